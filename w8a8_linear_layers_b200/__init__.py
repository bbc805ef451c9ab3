"""Python binding of libw8a8.so, the B200 (sm_100a) SmoothQuant-style W8A8
linear layer.

Argument marshalling only: every function here has the name and the meaning
of the C entry point declared in include/w8a8.h, takes torch CUDA tensors
(the caller owns them; outputs are written in place), passes their device
pointers and the current CUDA stream, and raises W8A8Error on a non-OK status.
All computation happens in the library's CUDA kernels; there is no CPU or
PyTorch fallback, and importing fails loudly if the library is missing.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# W8A8_LIBRARY=debug loads the debug build (libw8a8_debug.so: the kernels
# count non-finite inputs and failed index checks, see sq_debug_status)
LIB_PATH = os.path.join(_HERE, "libw8a8_debug.so" if os.environ.get("W8A8_LIBRARY") == "debug" else "libw8a8.so")

SQ_F32, SQ_BF16 = 0, 1
STATUS = ["SQ_OK", "SQ_ERR_NULL", "SQ_ERR_SHAPE", "SQ_ERR_DTYPE", "SQ_ERR_ALIGN", "SQ_ERR_ARG",
          "SQ_ERR_UNSUPPORTED", "SQ_ERR_CUDA", "SQ_ERR_DEVICE"]

# every symbol include/w8a8.h declares
EXPORTS = ["sq_status_string", "sq_last_error_detail", "sq_abi_version", "sq_device_fault",
           "sq_selftest_bounded_wait",
           "sq_calib_absmax", "sq_smooth_fold", "ssz_quant_weight", "quant_act_per_token",
           "w8a8_gemm_dequant", "sq_static_range_update", "quant_act_static", "quant_act_per_token_rowsum",
           "ssz_quant_weight_asym", "w8a8_gemm_dequant_asym", "sq_pack_int4", "w4a8_gemm_dequant",
           "sq_layernorm_quant", "quant_act_given_scale", "sq_dequant", "sq_smooth_factor", "sq_debug_status"]


class W8A8Error(RuntimeError):
    def __init__(self, fn: str, status: int, detail: str):
        self.status = status
        self.status_name = STATUS[status] if 0 <= status < len(STATUS) else "SQ_ERR_UNKNOWN"
        self.detail = detail
        super().__init__("%s failed: %s (%s)" % (fn, self.status_name, detail))


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            "%s is not built; run `python w8a8_linear_layers_b200/build.py`" % LIB_PATH)
    lib = ctypes.CDLL(LIB_PATH)
    P, I64, I, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
    sig = {
        "sq_status_string": ([I], ctypes.c_char_p),
        "sq_last_error_detail": ([], ctypes.c_char_p),
        "sq_abi_version": ([], I),
        "sq_device_fault": ([P, P], I),
        "sq_selftest_bounded_wait": ([ctypes.c_uint32, P], I),
        "sq_calib_absmax": ([P, I, I64, I64, P, I, P], I),
        "sq_smooth_fold": ([P, P, I, I64, I64, F, P, P, P, P, P], I),
        "sq_smooth_factor": ([P, P, I64, F, P, P, P], I),
        "ssz_quant_weight": ([P, I, I64, I64, P, I, I, P, P, P, P, P], I),
        "quant_act_per_token": ([P, I, I64, I64, P, P, P, P], I),
        "w8a8_gemm_dequant": ([P, P, P, P, I64, I64, I64, P, I, P, P], I),
        "sq_static_range_update": ([P, P, I64, F, I, P, P], I),
        "quant_act_static": ([P, I, I64, I64, P, P, P, P, P, P], I),
        "quant_act_per_token_rowsum": ([P, I, I64, I64, P, P, P, P, P], I),
        "ssz_quant_weight_asym": ([P, I, I64, I64, P, I, P, P, P, P, P, P], I),
        "w8a8_gemm_dequant_asym": ([P, P, P, P, P, P, I64, I64, I64, P, I, P, P], I),
        "sq_pack_int4": ([P, I64, I64, P, P], I),
        "sq_layernorm_quant": ([P, I, I64, I64, P, P, F, P, P, P, P], I),
        "quant_act_given_scale": ([P, I, I64, I64, P, P, P, P], I),
        "sq_dequant": ([P, P, P, I64, I64, P, I, P], I),
        "w4a8_gemm_dequant": ([P, P, P, P, I64, I64, I64, P, I, P, P], I),
        "sq_debug_status": ([P, P, P, P], I),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


lib = _load()


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise W8A8Error(fn, status, lib.sq_last_error_detail().decode())


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor, got one on %s" % t.device)
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return SQ_F32
    if t.dtype == torch.bfloat16:
        return SQ_BF16
    raise ValueError("unsupported dtype %s (float32 or bfloat16)" % t.dtype)


def _need(t: torch.Tensor | None, dtype: torch.dtype, name: str) -> None:
    if t is not None and t.dtype != dtype:
        raise ValueError("%s must be %s, got %s" % (name, dtype, t.dtype))


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def abi_version() -> int:
    return lib.sq_abi_version()


def debug_status(stream=None) -> tuple[int, int, bool]:
    """(non-finite inputs, failed index checks, debug build?) counted since the
    last call, read and cleared (sq_debug_status; zeros in a release build)."""
    nf, ix, en = ctypes.c_uint64(0), ctypes.c_uint64(0), ctypes.c_int(0)
    _check("sq_debug_status", lib.sq_debug_status(_stream(stream), ctypes.byref(nf), ctypes.byref(ix),
                                                  ctypes.byref(en)))
    return int(nf.value), int(ix.value), bool(en.value)


def device_fault(stream=None) -> int:
    """Read and clear the device fault word (0: no kernel gave up on a wait)."""
    out = ctypes.c_uint32(0)
    _check("sq_device_fault", lib.sq_device_fault(_stream(stream), ctypes.byref(out)))
    return out.value


def selftest_bounded_wait(limit_ms: int = 50, stream=None) -> None:
    """Launch the bounded-wait self test (see include/w8a8.h)."""
    _check("sq_selftest_bounded_wait", lib.sq_selftest_bounded_wait(int(limit_ms), _stream(stream)))


def sq_calib_absmax(x: torch.Tensor, absmax: torch.Tensor, accumulate: bool = False, stream=None) -> None:
    """absmax[j] = max(accumulate ? absmax[j] : 0, max_t |x[t,j]|)."""
    _need(absmax, torch.float32, "absmax")
    M, K = x.shape
    _check("sq_calib_absmax", lib.sq_calib_absmax(_ptr(x), _dtype(x), M, K, _ptr(absmax),
                                                   1 if accumulate else 0, _stream(stream)))


def sq_smooth_fold(x_absmax: torch.Tensor, w: torch.Tensor, alpha: float, w_absmax_out: torch.Tensor,
                   s_out: torch.Tensor, inv_s_out: torch.Tensor, w_folded_out: torch.Tensor | None = None,
                   stream=None) -> None:
    """Weight column absmax, s = ax^alpha / aw^(1-alpha), 1/s, optional W diag(s)."""
    for t, n in ((x_absmax, "x_absmax"), (w_absmax_out, "w_absmax_out"), (s_out, "s_out"),
                 (inv_s_out, "inv_s_out"), (w_folded_out, "w_folded_out")):
        _need(t, torch.float32, n)
    N, K = w.shape
    _check("sq_smooth_fold", lib.sq_smooth_fold(_ptr(x_absmax), _ptr(w), _dtype(w), N, K, float(alpha),
                                                 _ptr(w_absmax_out), _ptr(s_out), _ptr(inv_s_out),
                                                 _ptr(w_folded_out), _stream(stream)))


def sq_smooth_factor(x_absmax: torch.Tensor, w_absmax: torch.Tensor, alpha: float, s_out: torch.Tensor,
                     inv_s_out: torch.Tensor, stream=None) -> None:
    """s = ax^alpha / aw^(1-alpha) and 1/s from both abs-max vectors (w_absmax:
    sq_calib_absmax of the weight), as sq_smooth_fold computes them."""
    for t, n in ((x_absmax, "x_absmax"), (w_absmax, "w_absmax"), (s_out, "s_out"), (inv_s_out, "inv_s_out")):
        _need(t, torch.float32, n)
    K = x_absmax.numel()
    if w_absmax.numel() != K or s_out.numel() != K or inv_s_out.numel() != K:
        raise ValueError("x_absmax, w_absmax, s_out and inv_s_out must all hold K values")
    _check("sq_smooth_factor", lib.sq_smooth_factor(_ptr(x_absmax), _ptr(w_absmax), K, float(alpha), _ptr(s_out),
                                                     _ptr(inv_s_out), _stream(stream)))


def ssz_quant_weight(w: torch.Tensor, s: torch.Tensor | None, bits: int, max_iters: int, q_out: torch.Tensor,
                     scale_out: torch.Tensor, mse_out: torch.Tensor | None = None,
                     iters_out: torch.Tensor | None = None, stream=None) -> None:
    """SSZ per-output-channel symmetric quantization of w [N,K] (folded by s)."""
    _need(s, torch.float32, "s")
    _need(q_out, torch.int8, "q_out")
    _need(scale_out, torch.float32, "scale_out")
    _need(mse_out, torch.float64, "mse_out")
    _need(iters_out, torch.int32, "iters_out")
    N, K = w.shape
    _check("ssz_quant_weight", lib.ssz_quant_weight(_ptr(w), _dtype(w), N, K, _ptr(s), int(bits), int(max_iters),
                                                     _ptr(q_out), _ptr(scale_out), _ptr(mse_out),
                                                     _ptr(iters_out), _stream(stream)))


def quant_act_per_token(x: torch.Tensor, inv_s: torch.Tensor | None, q_out: torch.Tensor,
                        scale_out: torch.Tensor, stream=None) -> None:
    """Per-token int8 codes and scales of x * inv_s."""
    _need(inv_s, torch.float32, "inv_s")
    _need(q_out, torch.int8, "q_out")
    _need(scale_out, torch.float32, "scale_out")
    M, K = x.shape
    _check("quant_act_per_token", lib.quant_act_per_token(_ptr(x), _dtype(x), M, K, _ptr(inv_s), _ptr(q_out),
                                                           _ptr(scale_out), _stream(stream)))


def quant_act_per_token_rowsum(x: torch.Tensor, inv_s: torch.Tensor | None, q_out: torch.Tensor,
                               scale_out: torch.Tensor, rowsum_out: torch.Tensor, stream=None) -> None:
    """quant_act_per_token plus the exact row sums of the codes (int32)."""
    _need(inv_s, torch.float32, "inv_s")
    _need(q_out, torch.int8, "q_out")
    _need(scale_out, torch.float32, "scale_out")
    _need(rowsum_out, torch.int32, "rowsum_out")
    M, K = x.shape
    _check("quant_act_per_token_rowsum",
           lib.quant_act_per_token_rowsum(_ptr(x), _dtype(x), M, K, _ptr(inv_s), _ptr(q_out), _ptr(scale_out),
                                          _ptr(rowsum_out), _stream(stream)))


def ssz_quant_weight_asym(w: torch.Tensor, s: torch.Tensor | None, max_iters: int, q_out: torch.Tensor,
                          scale_out: torch.Tensor, offset_out: torch.Tensor, mse_out: torch.Tensor | None = None,
                          iters_out: torch.Tensor | None = None, stream=None) -> None:
    """Asymmetric per-channel int8 SSZ: w * s ~ scale * (q + 128) + offset."""
    _need(s, torch.float32, "s")
    _need(q_out, torch.int8, "q_out")
    _need(scale_out, torch.float32, "scale_out")
    _need(offset_out, torch.float32, "offset_out")
    _need(mse_out, torch.float64, "mse_out")
    _need(iters_out, torch.int32, "iters_out")
    N, K = w.shape
    _check("ssz_quant_weight_asym",
           lib.ssz_quant_weight_asym(_ptr(w), _dtype(w), N, K, _ptr(s), int(max_iters), _ptr(q_out),
                                     _ptr(scale_out), _ptr(offset_out), _ptr(mse_out), _ptr(iters_out),
                                     _stream(stream)))


def w8a8_gemm_dequant_asym(qx: torch.Tensor, sx: torch.Tensor, rowsum: torch.Tensor, qw: torch.Tensor,
                           sw: torch.Tensor, ow: torch.Tensor, y: torch.Tensor, acc_out: torch.Tensor | None = None,
                           stream=None) -> None:
    """GEMM + dequant with asymmetric weights (scale sw, offset ow)."""
    _need(qx, torch.int8, "qx")
    _need(qw, torch.int8, "qw")
    _need(sx, torch.float32, "sx")
    _need(sw, torch.float32, "sw")
    _need(ow, torch.float32, "ow")
    _need(rowsum, torch.int32, "rowsum")
    _need(acc_out, torch.int32, "acc_out")
    M, K = qx.shape
    N = qw.shape[0]
    _check("w8a8_gemm_dequant_asym",
           lib.w8a8_gemm_dequant_asym(_ptr(qx), _ptr(sx), _ptr(rowsum), _ptr(qw), _ptr(sw), _ptr(ow), M, N, K,
                                      _ptr(y), _dtype(y), _ptr(acc_out), _stream(stream)))


def sq_layernorm_quant(h: torch.Tensor, gamma: torch.Tensor | None, beta: torch.Tensor | None, eps: float,
                       inv_s: torch.Tensor | None, q_out: torch.Tensor, scale_out: torch.Tensor, stream=None) -> None:
    """LayerNorm of h, times inv_s, as per-token int8 codes and scales."""
    _need(gamma, torch.float32, "gamma")
    _need(beta, torch.float32, "beta")
    _need(inv_s, torch.float32, "inv_s")
    _need(q_out, torch.int8, "q_out")
    _need(scale_out, torch.float32, "scale_out")
    M, K = h.shape
    _check("sq_layernorm_quant", lib.sq_layernorm_quant(_ptr(h), _dtype(h), M, K, _ptr(gamma), _ptr(beta),
                                                         float(eps), _ptr(inv_s), _ptr(q_out), _ptr(scale_out),
                                                         _stream(stream)))


def quant_act_given_scale(x: torch.Tensor, inv_s: torch.Tensor | None, sx: torch.Tensor, q_out: torch.Tensor,
                          stream=None) -> None:
    """int8 codes of x * inv_s at the given per-row scales sx."""
    _need(inv_s, torch.float32, "inv_s")
    _need(sx, torch.float32, "sx")
    _need(q_out, torch.int8, "q_out")
    M, K = x.shape
    _check("quant_act_given_scale", lib.quant_act_given_scale(_ptr(x), _dtype(x), M, K, _ptr(inv_s), _ptr(sx),
                                                               _ptr(q_out), _stream(stream)))


def sq_dequant(acc: torch.Tensor, sx: torch.Tensor, sw: torch.Tensor, y: torch.Tensor, stream=None) -> None:
    """y = ((float)acc * sx[row]) * sw[col] from int32 accumulators."""
    _need(acc, torch.int32, "acc")
    _need(sx, torch.float32, "sx")
    _need(sw, torch.float32, "sw")
    M, N = acc.shape
    _check("sq_dequant", lib.sq_dequant(_ptr(acc), _ptr(sx), _ptr(sw), M, N, _ptr(y), _dtype(y), _stream(stream)))


def sq_pack_int4(q: torch.Tensor, packed: torch.Tensor, stream=None) -> None:
    """Two int4 codes per byte (element 2i in the low nibble)."""
    _need(q, torch.int8, "q")
    _need(packed, torch.uint8, "packed")
    N, K = q.shape
    _check("sq_pack_int4", lib.sq_pack_int4(_ptr(q), N, K, _ptr(packed), _stream(stream)))


def w4a8_gemm_dequant(qx: torch.Tensor, sx: torch.Tensor, qw4: torch.Tensor, sw: torch.Tensor, y: torch.Tensor,
                      acc_out: torch.Tensor | None = None, stream=None) -> None:
    """GEMM + dequant with packed int4 weight codes qw4 [N, K/2]."""
    _need(qx, torch.int8, "qx")
    _need(qw4, torch.uint8, "qw4")
    _need(sx, torch.float32, "sx")
    _need(sw, torch.float32, "sw")
    _need(acc_out, torch.int32, "acc_out")
    M, K = qx.shape
    N = qw4.shape[0]
    _check("w4a8_gemm_dequant", lib.w4a8_gemm_dequant(_ptr(qx), _ptr(sx), _ptr(qw4), _ptr(sw), M, N, K, _ptr(y),
                                                       _dtype(y), _ptr(acc_out), _stream(stream)))


STATIC_RANGE_RATE = 0.9  # moving rate of the static activation range (not given by the pages)


def sq_static_range_update(x_absmax: torch.Tensor, inv_s: torch.Tensor | None, range_: torch.Tensor,
                           first: bool, rate: float = STATIC_RANGE_RATE, stream=None) -> None:
    """Blend one calibration batch (its per-channel abs-max) into the static
    activation range held in range_ (one fp32 on the device)."""
    _need(x_absmax, torch.float32, "x_absmax")
    _need(inv_s, torch.float32, "inv_s")
    _need(range_, torch.float32, "range")
    K = x_absmax.shape[0]
    _check("sq_static_range_update", lib.sq_static_range_update(_ptr(x_absmax), _ptr(inv_s), K, float(rate),
                                                                 1 if first else 0, _ptr(range_), _stream(stream)))


def quant_act_static(x: torch.Tensor, inv_s: torch.Tensor | None, range_: torch.Tensor, q_out: torch.Tensor,
                     scale_out: torch.Tensor | None = None, rowsum_out: torch.Tensor | None = None,
                     stream=None) -> None:
    """int8 codes of x * inv_s at the static scale range_/127 (saturating)."""
    _need(inv_s, torch.float32, "inv_s")
    _need(range_, torch.float32, "range")
    _need(q_out, torch.int8, "q_out")
    _need(scale_out, torch.float32, "scale_out")
    _need(rowsum_out, torch.int32, "rowsum_out")
    M, K = x.shape
    _check("quant_act_static", lib.quant_act_static(_ptr(x), _dtype(x), M, K, _ptr(inv_s), _ptr(range_),
                                                     _ptr(q_out), _ptr(scale_out), _ptr(rowsum_out),
                                                     _stream(stream)))


def w8a8_gemm_dequant(qx: torch.Tensor, sx: torch.Tensor, qw: torch.Tensor, sw: torch.Tensor, y: torch.Tensor,
                      acc_out: torch.Tensor | None = None, stream=None) -> None:
    """y = ((float)(qx @ qw^T) * sx[:,None]) * sw[None,:], int32 accumulation."""
    _need(qx, torch.int8, "qx")
    _need(qw, torch.int8, "qw")
    _need(sx, torch.float32, "sx")
    _need(sw, torch.float32, "sw")
    _need(acc_out, torch.int32, "acc_out")
    M, K = qx.shape
    N, K2 = qw.shape
    if K != K2 or tuple(y.shape) != (M, N):
        raise ValueError("shape mismatch: qx %s, qw %s, y %s" % (tuple(qx.shape), tuple(qw.shape), tuple(y.shape)))
    _check("w8a8_gemm_dequant", lib.w8a8_gemm_dequant(_ptr(qx), _ptr(sx), _ptr(qw), _ptr(sw), M, N, K, _ptr(y),
                                                       _dtype(y), _ptr(acc_out), _stream(stream)))


class W8A8Linear:
    """A calibrated SmoothQuant W8A8 linear layer built from the library calls.

    calibrate(x) accumulates the activation absmax; quantize() smooths and
    SSZ-quantizes the weight; forward(x) quantizes x and runs the integer GEMM
    with the fused dequant.  Options (the next rows of the path):
      weights="sym8"  symmetric int8 SSZ (default), "asym8" asymmetric int8
                      SSZ (scale and offset), "int4" int4 SSZ packed two per
                      byte with the W4A8 GEMM;
      act_scales="dynamic" per-token scales (default) or "static": a
                      per-tensor range, the moving average of each
                      calibration batch's abs-max (calibrate_static(x) after
                      quantize()).
    forward_ln(h, gamma, beta, eps) applies the LayerNorm that produces x,
    the smoothing and the per-token quantization in one kernel.  Buffers are
    torch tensors on the weight's device (memory plumbing only)."""

    def __init__(self, w: torch.Tensor, alpha: float = 0.5, bits: int = 8, max_iters: int = 20,
                 out_dtype: torch.dtype | None = None, weights: str = "sym8", act_scales: str = "dynamic",
                 static_rate: float = 0.9):
        if weights not in ("sym8", "asym8", "int4"):
            raise ValueError("weights must be sym8, asym8 or int4")
        if act_scales not in ("dynamic", "static"):
            raise ValueError("act_scales must be dynamic or static")
        if weights == "int4":
            bits = 4
        self.w = w.contiguous()
        self.N, self.K = w.shape
        self.alpha, self.bits, self.max_iters = alpha, bits, max_iters
        self.weights, self.act_scales, self.static_rate = weights, act_scales, static_rate
        self.out_dtype = out_dtype or w.dtype
        dev = w.device
        f32 = dict(device=dev, dtype=torch.float32)
        self.ax = torch.zeros(self.K, **f32)
        self.aw = torch.empty(self.K, **f32)
        self.s = torch.empty(self.K, **f32)
        self.inv_s = torch.empty(self.K, **f32)
        self.qw = torch.empty(self.N, self.K, device=dev, dtype=torch.int8)
        self.sw = torch.empty(self.N, **f32)
        self.ow = torch.empty(self.N, **f32) if weights == "asym8" else None
        self.qw4 = torch.empty(self.N, self.K // 2, device=dev, dtype=torch.uint8) if weights == "int4" else None
        self.mse = torch.empty(self.N, device=dev, dtype=torch.float64)
        self.iters = torch.empty(self.N, device=dev, dtype=torch.int32)
        self.range = torch.zeros(1, **f32)
        self._calibrated = False
        self._static_batches = 0

    def calibrate(self, x: torch.Tensor) -> None:
        sq_calib_absmax(x, self.ax, accumulate=self._calibrated)
        self._calibrated = True

    def quantize(self) -> None:
        sq_smooth_fold(self.ax, self.w, self.alpha, self.aw, self.s, self.inv_s)
        if self.weights == "asym8":
            ssz_quant_weight_asym(self.w, self.s, self.max_iters, self.qw, self.sw, self.ow, self.mse, self.iters)
        else:
            ssz_quant_weight(self.w, self.s, self.bits, self.max_iters, self.qw, self.sw, self.mse, self.iters)
        if self.weights == "int4":
            sq_pack_int4(self.qw, self.qw4)

    def calibrate_static(self, x: torch.Tensor) -> None:
        """Blend one calibration batch into the static activation range
        (after quantize(): the range is of x * inv_s)."""
        axb = torch.empty(self.K, device=x.device, dtype=torch.float32)
        sq_calib_absmax(x, axb)
        sq_static_range_update(axb, self.inv_s, self.range, first=self._static_batches == 0, rate=self.static_rate)
        self._static_batches += 1

    def _gemm(self, qx, sx, rs, y):
        if self.weights == "asym8":
            w8a8_gemm_dequant_asym(qx, sx, rs, self.qw, self.sw, self.ow, y)
        elif self.weights == "int4":
            w4a8_gemm_dequant(qx, sx, self.qw4, self.sw, y)
        else:
            w8a8_gemm_dequant(qx, sx, self.qw, self.sw, y)

    def _forward_into(self, x, qx, sx, rs, y) -> None:
        """The per-inference kernels into caller buffers: codes qx [M, K],
        scales sx [M], row sums rs [M] (asym8 only, else None), output y."""
        if self.act_scales == "static":
            if self._static_batches == 0:
                raise RuntimeError("static activation scales need calibrate_static() first")
            quant_act_static(x, self.inv_s, self.range, qx, sx, rs)
        else:
            quant_act_per_token_rowsum(x, self.inv_s, qx, sx, rs)
        self._gemm(qx, sx, rs, y)

    def forward(self, x: torch.Tensor, y: torch.Tensor | None = None) -> torch.Tensor:
        M = x.shape[0]
        qx = torch.empty(M, self.K, device=x.device, dtype=torch.int8)
        sx = torch.empty(M, device=x.device, dtype=torch.float32)
        rs = torch.empty(M, device=x.device, dtype=torch.int32) if self.weights == "asym8" else None
        if y is None:
            y = torch.empty(M, self.N, device=x.device, dtype=self.out_dtype)
        self._forward_into(x, qx, sx, rs, y)
        return y

    def forward_host(self, x_host: torch.Tensor, y_host: torch.Tensor, chunk_rows: int = 2048,
                     streamer: "HostStreamer | None" = None) -> None:
        """forward() on activations in pinned host memory: y_host [M, N]
        (pinned, out_dtype) receives the output, the copies in and out
        overlapped with the kernels chunk by chunk (HostStreamer; pass one
        to reuse its device buffers).  Returns once enqueued: synchronize the
        current stream before reading y_host."""
        st = streamer or HostStreamer(self.w.device, chunk_rows, self.K, self.N, x_host.dtype, self.out_dtype)
        # the kernels of all chunks run in order on one stream, so one
        # row-sum buffer serves them all
        rs = torch.empty(st.rows, device=self.w.device, dtype=torch.int32) if self.weights == "asym8" else None

        def fn(x, qx, sx, y):
            self._forward_into(x, qx, sx, None if rs is None else rs[: x.shape[0]], y)

        st.run([(x_host, y_host, fn)])

    def graphed(self, M: int, x_dtype: torch.dtype | None = None) -> "GraphedLinear":
        """forward() for M-token inputs captured in a CUDA graph (see
        GraphedLinear)."""
        return GraphedLinear(self, M, x_dtype or self.w.dtype)

    def forward_ln(self, h: torch.Tensor, gamma: torch.Tensor | None, beta: torch.Tensor | None,
                   eps: float = 1e-5, y: torch.Tensor | None = None) -> torch.Tensor:
        """forward(LayerNorm(h)) with the LayerNorm, the smoothing and the
        per-token quantization fused (dynamic scales, sym8 or int4 weights)."""
        if self.weights == "asym8" or self.act_scales == "static":
            raise ValueError("forward_ln supports dynamic scales with sym8 or int4 weights")
        M = h.shape[0]
        qx = torch.empty(M, self.K, device=h.device, dtype=torch.int8)
        sx = torch.empty(M, device=h.device, dtype=torch.float32)
        sq_layernorm_quant(h, gamma, beta, eps, self.inv_s, qx, sx)
        if y is None:
            y = torch.empty(M, self.N, device=h.device, dtype=self.out_dtype)
        self._gemm(qx, sx, None, y)
        return y


class GraphedLinear:
    """A W8A8Linear's forward for M-token inputs captured once in a CUDA graph
    (the activation quantization and the GEMM, two kernels): write the input
    into .x, call replay(), read .y.  Built by W8A8Linear.graphed(M); the
    layer must be quantized (and, for static scales, calibrated) first."""

    def __init__(self, lin: "W8A8Linear", M: int, x_dtype: torch.dtype):
        dev = lin.w.device
        self.x = torch.zeros(M, lin.K, device=dev, dtype=x_dtype)
        self.y = torch.empty(M, lin.N, device=dev, dtype=lin.out_dtype)
        self._lin = lin
        stream = torch.cuda.Stream(device=dev)
        stream.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(stream):
            lin.forward(self.x, self.y)  # one eager call: one-time kernel attributes are set outside the capture
        torch.cuda.current_stream(dev).wait_stream(stream)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            lin.forward(self.x, self.y)

    def replay(self) -> torch.Tensor:
        self.graph.replay()
        return self.y


from .host import HostStreamer  # noqa: E402  (pinned-host linears with overlapped copies)
