"""ctypes binding of libsvdq.so (include/svdq.h). Argument marshalling only: every step of the layer
runs in the library's CUDA kernels; torch provides device memory and the current stream.

There is no fallback: if the library is missing or the device is not sm_100a, the calls raise.
"""
from __future__ import annotations

import ctypes
import os
import re
from ctypes import POINTER, byref, c_char_p, c_int, c_size_t, c_ulonglong, c_void_p

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsvdq.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "svdq.h")

EPI_NONE, EPI_BIAS, EPI_SWIGLU, EPI_BIAS_SWIGLU = 0, 1, 2, 3
OUT_BF16, OUT_F32 = 0, 1
STATUS_NAMES = {0: "SVDQ_OK", 1: "SVDQ_ERR_INVALID_ARG", 2: "SVDQ_ERR_UNSUPPORTED", 3: "SVDQ_ERR_CUDA",
                4: "SVDQ_ERR_TIMEOUT"}


class SvdqWeight(ctypes.Structure):
    _fields_ = [("N", c_int), ("K", c_int), ("r", c_int), ("swiglu_interleaved", c_int), ("n_tile", c_int),
                ("reserved0", c_int), ("codes", c_void_p), ("scales", c_void_p), ("g_w", c_void_p),
                ("inv_lambda", c_void_p), ("L1s_t", c_void_p), ("L2_t", c_void_p), ("tmap", c_ulonglong * 32)]


class SvdqAct(ctypes.Structure):
    _fields_ = [("M", c_int), ("K", c_int), ("r", c_int), ("M_pad", c_int), ("codes", c_void_p),
                ("scales", c_void_p), ("U", c_void_p), ("alpha", c_void_p)]


class SvdqFp8rWeight(ctypes.Structure):
    _fields_ = [("N", c_int), ("K", c_int), ("r", c_int), ("swiglu_interleaved", c_int), ("n_tile", c_int),
                ("reserved0", c_int), ("codes", c_void_p), ("row_scale", c_void_p), ("inv_lambda", c_void_p),
                ("L1s_t", c_void_p), ("L2_t", c_void_p), ("tmap", c_ulonglong * 32)]


class SvdqFp8rAct(ctypes.Structure):
    _fields_ = [("M", c_int), ("K", c_int), ("r", c_int), ("M_pad", c_int), ("codes", c_void_p),
                ("row_scale", c_void_p), ("row_rscale", c_void_p), ("U", c_void_p)]


class SvdqError(RuntimeError):
    def __init__(self, func: str, status: int, message: str):
        super().__init__(f"{func}: {STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


_lib = None


def _declare(lib):
    W, A = POINTER(SvdqWeight), POINTER(SvdqAct)
    FW, FA = POINTER(SvdqFp8rWeight), POINTER(SvdqFp8rAct)
    sig = {
        "svdq_fp8r_weight_bytes": (c_size_t, [c_int, c_int, c_int]),
        "svdq_fp8r_act_bytes": (c_size_t, [c_int, c_int, c_int]),
        "svdq_fp8r_pack_weight": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int,
                                          c_void_p, c_size_t, FW, c_void_p]),
        "svdq_fp8r_act_bind": (c_int, [c_int, c_int, c_int, c_void_p, c_size_t, FA]),
        "svdq_fp8r_quantize_act": (c_int, [c_void_p, FW, FA, c_void_p]),
        "svdq_fp8r_gemm": (c_int, [FA, FW, c_void_p, c_int, c_void_p, c_int, c_void_p]),
        "svdq_fp8r_export_weight": (c_int, [FW, c_void_p, c_void_p, c_void_p]),
        "svdq_fp8r_export_act": (c_int, [FA, c_void_p, c_void_p, c_void_p]),
        "svdq_mlp_scratch_bytes": (c_size_t, [c_int, c_int]),
        "svdq_gemm_swiglu_quant": (c_int, [A, W, c_void_p, W, c_void_p, A, c_void_p, c_size_t, c_void_p, c_void_p]),
        "svdq_gemm_swiglu_quant_noscratch": (c_int, [A, W, c_void_p, W, c_void_p, A, c_void_p, c_void_p]),
        "svdq_weight_bytes": (c_size_t, [c_int, c_int, c_int]),
        "svdq_act_bytes": (c_size_t, [c_int, c_int, c_int]),
        "svdq_weight_bytes_tiled": (c_size_t, [c_int, c_int, c_int, c_int]),
        "svdq_pack_weight": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_void_p,
                                     c_size_t, W, c_void_p]),
        "svdq_act_bind": (c_int, [c_int, c_int, c_int, c_void_p, c_size_t, A]),
        "svdq_weight_bind": (c_int, [c_int, c_int, c_int, c_int, c_int, c_void_p, c_size_t, W]),
        "svdq_calibrate_act": (c_int, [c_void_p, c_int, W, c_void_p, c_void_p]),
        "svdq_quantize_act": (c_int, [c_void_p, W, c_void_p, A, c_void_p]),
        "svdq_gemm": (c_int, [A, W, c_void_p, c_int, c_void_p, c_int, c_void_p]),
        "svdq_export_weight": (c_int, [W, c_void_p, c_void_p, c_void_p]),
        "svdq_export_act": (c_int, [A, c_void_p, c_void_p, c_void_p]),
        "svdq_device_status": (c_int, [c_int]),
        "svdq_watchdog_selftest": (c_int, [c_ulonglong, c_void_p]),
        "svdq_set_wait_limit_ns": (c_int, [c_ulonglong]),
        "svdq_status_str": (c_char_p, [c_int]),
        "svdq_last_error": (c_char_p, []),
        "svdq_abi_version": (c_int, []),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args


def lib():
    """The loaded library. Raises if libsvdq.so has not been built (no fallback exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -c 'import __graft_entry__ as g; "
                               "g.build()'` (nvcc, sm_100a)")
        l = ctypes.CDLL(LIB_PATH)
        _declare(l)
        _lib = l
    return _lib


def header_functions() -> list[str]:
    """Names of the entry points include/svdq.h declares."""
    with open(HEADER) as f:
        return sorted(set(re.findall(r"^SVDQ_API\s+[\w\s\*]+?\b(svdq_\w+)\s*\(", f.read(), re.M)))


def _check(func: str, status: int):
    if status != 0:
        raise SvdqError(func, status, lib().svdq_last_error().decode())


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _ptr(t):
    return None if t is None else c_void_p(t.data_ptr())


def _need(t, dtype, name, ndim=None):
    if t.dtype != dtype or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous CUDA {dtype} tensor, got {t.dtype} on {t.device}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name}: expected {ndim} dims, got {tuple(t.shape)}")


class PackedWeight:
    """One layer's packed weight (device buffer + svdq_weight descriptor)."""

    def __init__(self, R: torch.Tensor, L1s: torch.Tensor | None, L2: torch.Tensor | None,
                 inv_lambda: torch.Tensor, swiglu: bool = False):
        _need(R, torch.float32, "R", 2)
        _need(inv_lambda, torch.float32, "inv_lambda", 1)
        N, K = R.shape
        r = 0 if L1s is None else L1s.shape[1]
        if r:
            _need(L1s, torch.bfloat16, "L1s", 2)
            _need(L2, torch.bfloat16, "L2", 2)
            if tuple(L1s.shape) != (K, r) or tuple(L2.shape) != (r, N):
                raise ValueError("L1s must be [K, r] and L2 [r, N]")
        nbytes = lib().svdq_weight_bytes(N, K, r)
        if nbytes == 0:
            raise SvdqError("svdq_weight_bytes", 2, f"unsupported shape N={N} K={K} r={r}")
        self.device = R.device
        self.buf = torch.empty(nbytes, dtype=torch.uint8, device=R.device)
        self.desc = SvdqWeight()
        with torch.cuda.device(R.device):
            _check("svdq_pack_weight", lib().svdq_pack_weight(
                _ptr(R), _ptr(L1s) if r else None, _ptr(L2) if r else None, _ptr(inv_lambda), N, K, r,
                1 if swiglu else 0, _ptr(self.buf), nbytes, byref(self.desc), _stream(R.device)))
        self.N, self.K, self.r, self.swiglu = N, K, r, swiglu

    @property
    def n_tile(self) -> int:
        return self.desc.n_tile

    def state_dict(self) -> dict:
        """The packed blob (on the host) and the shape fields needed to re-bind it: a checkpoint of
        the quantized weight that does not need R, the branch factors or the pack kernels again."""
        return {"abi": lib().svdq_abi_version(), "N": self.N, "K": self.K, "r": self.r, "swiglu": self.swiglu,
                "n_tile": self.n_tile, "blob": self.buf.cpu()}

    @classmethod
    def from_state(cls, state: dict, device) -> "PackedWeight":
        """A packed weight from state_dict() output, copied to `device` and re-bound (its TMA
        descriptors re-encoded for the new address)."""
        if state["abi"] != lib().svdq_abi_version():
            raise ValueError(f"checkpoint ABI {state['abi']} != library ABI {lib().svdq_abi_version()}")
        blob = state["blob"]
        if not isinstance(blob, torch.Tensor) or blob.dtype != torch.uint8 or blob.dim() != 1 \
                or not blob.is_contiguous():
            raise ValueError("checkpoint blob: expected a contiguous one-dimensional uint8 tensor")
        need = lib().svdq_weight_bytes_tiled(state["N"], state["K"], state["r"], state["n_tile"])
        if need == 0 or blob.numel() != need:
            raise ValueError(f"checkpoint blob holds {blob.numel()} bytes; a weight packed with N={state['N']} "
                             f"K={state['K']} r={state['r']} n_tile={state['n_tile']} holds {need}")
        self = cls.__new__(cls)
        self.device = torch.device(device)
        self.buf = blob.to(self.device)
        self.desc = SvdqWeight()
        self.N, self.K, self.r, self.swiglu = state["N"], state["K"], state["r"], state["swiglu"]
        with torch.cuda.device(self.device):
            _check("svdq_weight_bind", lib().svdq_weight_bind(self.N, self.K, self.r, 1 if self.swiglu else 0,
                                                              state["n_tile"], _ptr(self.buf), self.buf.numel(),
                                                              byref(self.desc)))
        return self

    def g_w(self) -> torch.Tensor:
        off = self.desc.g_w - self.buf.data_ptr()
        return self.buf[off:off + 4].view(torch.float32)


class QuantizedAct:
    """A quantized activation buffer for M rows (codes, scales, U, alpha)."""

    def __init__(self, M: int, K: int, r: int, device):
        nbytes = lib().svdq_act_bytes(M, K, r)
        if nbytes == 0:
            raise SvdqError("svdq_act_bytes", 2, f"unsupported shape M={M} K={K} r={r}")
        self.buf = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.desc = SvdqAct()
        _check("svdq_act_bind", lib().svdq_act_bind(M, K, r, _ptr(self.buf), nbytes, byref(self.desc)))
        self.M, self.K, self.r, self.device = M, K, r, self.buf.device

    def _view(self, ptr, nbytes):
        off = ptr - self.buf.data_ptr()
        return self.buf[off:off + nbytes]

    def U(self) -> torch.Tensor:
        """[2, M_pad, r] bf16: the hi and lo halves of X L1s / alpha."""
        n = self.desc.M_pad * self.r
        return self._view(self.desc.U, 2 * n * 2).view(torch.bfloat16).view(2, self.desc.M_pad, self.r)

    def alpha(self) -> torch.Tensor:
        return self._view(self.desc.alpha, 4).view(torch.float32)


def calibrate_act(X: torch.Tensor, w: PackedWeight, out: torch.Tensor | None = None) -> torch.Tensor:
    """Static activation scale g_x (device fp32 [1]) from calibration data X [M, K] bf16."""
    _need(X, torch.bfloat16, "X", 2)
    out = torch.empty(1, dtype=torch.float32, device=X.device) if out is None else out
    with torch.cuda.device(X.device):
        _check("svdq_calibrate_act", lib().svdq_calibrate_act(_ptr(X), X.shape[0], byref(w.desc), _ptr(out),
                                                              _stream(X.device)))
    return out


def quantize_act(X: torch.Tensor, w: PackedWeight, g_x: torch.Tensor, act: QuantizedAct) -> QuantizedAct:
    """Kernel 1: smoothing + NVFP4 quantization + low-rank down-projection."""
    _need(X, torch.bfloat16, "X", 2)
    _need(g_x, torch.float32, "g_x")
    if X.shape[0] != act.M or X.shape[1] != w.K:
        raise ValueError("X shape does not match the act buffer / weight")
    with torch.cuda.device(X.device):
        _check("svdq_quantize_act", lib().svdq_quantize_act(_ptr(X), byref(w.desc), _ptr(g_x), byref(act.desc),
                                                            _stream(X.device)))
    return act


def gemm(act: QuantizedAct, w: PackedWeight, bias: torch.Tensor | None = None, epilogue: int | None = None,
         out_dtype=torch.bfloat16, out: torch.Tensor | None = None) -> torch.Tensor:
    """Kernel 2: NVFP4 GEMM + low-rank up-projection + bias / SwiGLU epilogue."""
    if epilogue is None:
        epilogue = (EPI_BIAS if bias is not None else EPI_NONE) | (EPI_SWIGLU if w.swiglu else 0)
    n_out = w.N // 2 if epilogue & EPI_SWIGLU else w.N
    if out is None:
        out = torch.empty(act.M, n_out, dtype=out_dtype, device=act.device)
    _need(out, out_dtype, "out", 2)
    if bias is not None:
        _need(bias, torch.bfloat16, "bias", 1)
    code = OUT_F32 if out_dtype == torch.float32 else OUT_BF16
    with torch.cuda.device(act.device):
        _check("svdq_gemm", lib().svdq_gemm(byref(act.desc), byref(w.desc), _ptr(bias), epilogue, _ptr(out), code,
                                            _stream(act.device)))
    return out


def linear(X, w, g_x=None, bias=None, act=None, out=None, out_dtype=torch.bfloat16):
    """The whole layer: kernel 1 then kernel 2 on the current stream. With g_x None the activation
    scale is computed from this X first (the dynamic mode: one extra amax pass over X)."""
    if g_x is None:
        g_x = calibrate_act(X, w)
    act = QuantizedAct(X.shape[0], w.K, w.r, X.device) if act is None else act
    quantize_act(X, w, g_x, act)
    return gemm(act, w, bias, out=out, out_dtype=out_dtype)


def export_weight(w: PackedWeight):
    codes = torch.empty(w.N, w.K // 2, dtype=torch.uint8, device=w.device)
    scales = torch.empty(w.N, w.K // 16, dtype=torch.uint8, device=w.device)
    with torch.cuda.device(w.device):
        _check("svdq_export_weight", lib().svdq_export_weight(byref(w.desc), _ptr(codes), _ptr(scales),
                                                              _stream(w.device)))
    return codes, scales


def export_act(act: QuantizedAct):
    codes = torch.empty(act.M, act.K // 2, dtype=torch.uint8, device=act.device)
    scales = torch.empty(act.M, act.K // 16, dtype=torch.uint8, device=act.device)
    with torch.cuda.device(act.device):
        _check("svdq_export_act", lib().svdq_export_act(byref(act.desc), _ptr(codes), _ptr(scales),
                                                        _stream(act.device)))
    return codes, scales


# ---------------------------------------------------------------- MLP chain with the down layer's
# kernel 1 fused into the gate/up GEMM's SwiGLU epilogue

def gemm_swiglu_quant(act: QuantizedAct, w: PackedWeight, bias, w_next: PackedWeight, g_x_next: torch.Tensor,
                      act_next: QuantizedAct, scratch: torch.Tensor | None = None,
                      h_out: torch.Tensor | None = None) -> QuantizedAct:
    """The gate/up GEMM with SwiGLU whose epilogue also quantizes h for the next layer (act_next);
    h itself is stored only into h_out (bf16 [M, N/2]) if given."""
    if not w.swiglu:
        raise ValueError("the gate/up weight must be packed with swiglu=True")
    _need(g_x_next, torch.float32, "g_x_next")
    if bias is not None:
        _need(bias, torch.bfloat16, "bias", 1)
    if h_out is not None:
        _need(h_out, torch.bfloat16, "h_out", 2)
    need = lib().svdq_mlp_scratch_bytes(act.M, w_next.r)
    if need == 0:
        raise SvdqError("svdq_mlp_scratch_bytes", 2, f"unsupported M={act.M} r_next={w_next.r}")
    if scratch is None:
        scratch = torch.empty(need, dtype=torch.uint8, device=act.device)
    with torch.cuda.device(act.device):
        _check("svdq_gemm_swiglu_quant", lib().svdq_gemm_swiglu_quant(
            byref(act.desc), byref(w.desc), _ptr(bias), byref(w_next.desc), _ptr(g_x_next), byref(act_next.desc),
            _ptr(scratch), scratch.numel(), _ptr(h_out), _stream(act.device)))
    return act_next


def gemm_swiglu_quant_noscratch(act: QuantizedAct, w: PackedWeight, bias, w_next: PackedWeight,
                                g_x_next: torch.Tensor, act_next: QuantizedAct,
                                h_out: torch.Tensor | None = None) -> QuantizedAct:
    """gemm_swiglu_quant for callers that cannot allocate: the partial sums of U' go to the
    library's built-in 8 MiB device buffer instead of a scratch tensor (nothing is allocated here or
    in the library). Calls on one device share that buffer: keep them ordered on one stream."""
    if not w.swiglu:
        raise ValueError("the gate/up weight must be packed with swiglu=True")
    _need(g_x_next, torch.float32, "g_x_next")
    if bias is not None:
        _need(bias, torch.bfloat16, "bias", 1)
    if h_out is not None:
        _need(h_out, torch.bfloat16, "h_out", 2)
    with torch.cuda.device(act.device):
        _check("svdq_gemm_swiglu_quant_noscratch", lib().svdq_gemm_swiglu_quant_noscratch(
            byref(act.desc), byref(w.desc), _ptr(bias), byref(w_next.desc), _ptr(g_x_next), byref(act_next.desc),
            _ptr(h_out), _stream(act.device)))
    return act_next


def mlp(X, w_up: PackedWeight, g_x_up, w_down: PackedWeight, g_x_down, bias_up=None, bias_down=None,
        out=None, out_dtype=torch.bfloat16):
    """The MLP chain X -> SwiGLU(X W_up^T + b_up) -> (.) W_down^T + b_down with the down layer's
    activation quantization done in the gate/up GEMM's epilogue (two GEMM launches, h stays on chip)."""
    act_up = quantize_act(X, w_up, g_x_up, QuantizedAct(X.shape[0], w_up.K, w_up.r, X.device))
    act_down = QuantizedAct(X.shape[0], w_down.K, w_down.r, X.device)
    gemm_swiglu_quant(act_up, w_up, bias_up, w_down, g_x_down, act_down)
    return gemm(act_down, w_down, bias_down, out=out, out_dtype=out_dtype)


# ---------------------------------------------------------------- row-wise FP8 (W8A8) variant

class Fp8rWeight:
    """One layer's weight packed for the row-wise FP8 path (E4M3 codes, one fp32 scale per row)."""

    def __init__(self, R: torch.Tensor, L1s: torch.Tensor | None, L2: torch.Tensor | None,
                 inv_lambda: torch.Tensor, swiglu: bool = False):
        _need(R, torch.float32, "R", 2)
        _need(inv_lambda, torch.float32, "inv_lambda", 1)
        N, K = R.shape
        r = 0 if L1s is None else L1s.shape[1]
        if r:
            _need(L1s, torch.bfloat16, "L1s", 2)
            _need(L2, torch.bfloat16, "L2", 2)
            if tuple(L1s.shape) != (K, r) or tuple(L2.shape) != (r, N):
                raise ValueError("L1s must be [K, r] and L2 [r, N]")
        nbytes = lib().svdq_fp8r_weight_bytes(N, K, r)
        if nbytes == 0:
            raise SvdqError("svdq_fp8r_weight_bytes", 2, f"unsupported shape N={N} K={K} r={r}")
        self.device = R.device
        self.buf = torch.empty(nbytes, dtype=torch.uint8, device=R.device)
        self.desc = SvdqFp8rWeight()
        with torch.cuda.device(R.device):
            _check("svdq_fp8r_pack_weight", lib().svdq_fp8r_pack_weight(
                _ptr(R), _ptr(L1s) if r else None, _ptr(L2) if r else None, _ptr(inv_lambda), N, K, r,
                1 if swiglu else 0, _ptr(self.buf), nbytes, byref(self.desc), _stream(R.device)))
        self.N, self.K, self.r, self.swiglu = N, K, r, swiglu


class Fp8rAct:
    """A row-wise FP8 activation buffer for M rows (codes, row scales, U)."""

    def __init__(self, M: int, K: int, r: int, device):
        nbytes = lib().svdq_fp8r_act_bytes(M, K, r)
        if nbytes == 0:
            raise SvdqError("svdq_fp8r_act_bytes", 2, f"unsupported shape M={M} K={K} r={r}")
        self.buf = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.desc = SvdqFp8rAct()
        _check("svdq_fp8r_act_bind", lib().svdq_fp8r_act_bind(M, K, r, _ptr(self.buf), nbytes, byref(self.desc)))
        self.M, self.K, self.r, self.device = M, K, r, self.buf.device


def quantize_act_fp8r(X: torch.Tensor, w: Fp8rWeight, act: Fp8rAct) -> Fp8rAct:
    """Row scales, then smoothing + E4M3 quantization + low-rank down-projection."""
    _need(X, torch.bfloat16, "X", 2)
    if X.shape[0] != act.M or X.shape[1] != w.K:
        raise ValueError("X shape does not match the act buffer / weight")
    with torch.cuda.device(X.device):
        _check("svdq_fp8r_quantize_act", lib().svdq_fp8r_quantize_act(_ptr(X), byref(w.desc), byref(act.desc),
                                                                      _stream(X.device)))
    return act


def gemm_fp8r(act: Fp8rAct, w: Fp8rWeight, bias: torch.Tensor | None = None, epilogue: int | None = None,
              out_dtype=torch.bfloat16, out: torch.Tensor | None = None) -> torch.Tensor:
    """FP8 GEMM + low-rank up-projection + bias / SwiGLU epilogue."""
    if epilogue is None:
        epilogue = (EPI_BIAS if bias is not None else EPI_NONE) | (EPI_SWIGLU if w.swiglu else 0)
    n_out = w.N // 2 if epilogue & EPI_SWIGLU else w.N
    if out is None:
        out = torch.empty(act.M, n_out, dtype=out_dtype, device=act.device)
    _need(out, out_dtype, "out", 2)
    if bias is not None:
        _need(bias, torch.bfloat16, "bias", 1)
    code = OUT_F32 if out_dtype == torch.float32 else OUT_BF16
    with torch.cuda.device(act.device):
        _check("svdq_fp8r_gemm", lib().svdq_fp8r_gemm(byref(act.desc), byref(w.desc), _ptr(bias), epilogue,
                                                      _ptr(out), code, _stream(act.device)))
    return out


def linear_fp8r(X, w: Fp8rWeight, bias=None, act=None, out=None, out_dtype=torch.bfloat16):
    """The whole row-wise FP8 layer on the current stream (the activation row scales always come
    from this X)."""
    act = Fp8rAct(X.shape[0], w.K, w.r, X.device) if act is None else act
    quantize_act_fp8r(X, w, act)
    return gemm_fp8r(act, w, bias, out=out, out_dtype=out_dtype)


def export_weight_fp8r(w: Fp8rWeight):
    codes = torch.empty(w.N, w.K, dtype=torch.uint8, device=w.device)
    scales = torch.empty(w.N, dtype=torch.float32, device=w.device)
    with torch.cuda.device(w.device):
        _check("svdq_fp8r_export_weight", lib().svdq_fp8r_export_weight(byref(w.desc), _ptr(codes), _ptr(scales),
                                                                        _stream(w.device)))
    return codes, scales


def export_act_fp8r(act: Fp8rAct):
    codes = torch.empty(act.M, act.K, dtype=torch.uint8, device=act.device)
    scales = torch.empty(act.M, dtype=torch.float32, device=act.device)
    with torch.cuda.device(act.device):
        _check("svdq_fp8r_export_act", lib().svdq_fp8r_export_act(byref(act.desc), _ptr(codes), _ptr(scales),
                                                                  _stream(act.device)))
    return codes, scales


def device_status(reset: bool = True) -> int:
    """Synchronizes; returns 0, or the SVDQ_ERR_TIMEOUT status if a bounded device wait ran out."""
    return lib().svdq_device_status(1 if reset else 0)


def watchdog_selftest(limit_ns: int, device=None):
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    with torch.cuda.device(device):
        _check("svdq_watchdog_selftest", lib().svdq_watchdog_selftest(limit_ns, _stream(device)))


def set_wait_limit_ns(ns: int):
    _check("svdq_set_wait_limit_ns", lib().svdq_set_wait_limit_ns(ns))


def last_error() -> str:
    return lib().svdq_last_error().decode()
