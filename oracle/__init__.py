"""Plain CPU oracle for the SmoothQuant-style W8A8 linear path.

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers.  The CUDA library never
imports, links or runs anything here, and nothing here imports the CUDA
package.  Every function takes and returns numpy arrays; bf16 data is passed
as its exact fp32 widening.

The arithmetic lives in ``oracle.c`` (plain C, built with -ffp-contract=off and
no fast-math); this module only marshals arrays.  Citations for each step are
in that file.  Every function here is pinned by ``tests/test_oracle_pins.py``
against invariants, closed forms, brute force and library routines.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
          "-fno-fast-math", "-fexcess-precision=standard"]

SSZ_CONVERGE_THRESHOLD = 1e-10
SSZ_MIN_SCALE = np.float32(1e-5)
SSZ_ITERS = 20


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc); returns the library path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None
_lib_path = None


def load_library(path: str | None) -> None:
    """Bind this module to another build of oracle.c (None: the default one).
    The mutation tests use it to run the pins against planted slips."""
    global _lib, _lib_path
    _lib, _lib_path = None, path


def build_variant(src_text: str, out_path: str) -> str:
    """Compile a modified copy of oracle.c (mutation tests) with the same flags."""
    src = out_path + ".c"
    with open(src, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", *CFLAGS, src, "-o", out_path, "-lm"])
    return out_path


def _L():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(_lib_path or build())
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        I = ctypes.c_int
        sig = {
            "oracle_calib_absmax": [P, I64, I64, P, I],
            "oracle_weight_col_absmax": [P, I64, I64, P],
            "oracle_smooth_factor": [P, P, I64, ctypes.c_float, P, P],
            "oracle_scale_columns": [P, I64, I64, P, P],
            "oracle_ssz_quant_weight": [P, I64, I64, I, I, P, P, P, P, P],
            "oracle_weight_codes": [P, I64, I64, I, P, P],
            "oracle_channel_mse": [P, I64, ctypes.c_float, I],
            "oracle_quant_act_per_token": [P, I64, I64, P, P, P],
            "oracle_gemm_i8": [P, P, I64, I64, I64, P],
            "oracle_dequant": [P, P, P, I64, I64, P, P],
            "oracle_static_batch_absmax": [P, I64, I64, P],
            "oracle_ssz_quant_weight_asym": [P, I64, I64, I, P, P, P, P, P, P],
            "oracle_channel_mse_asym": [P, I64, ctypes.c_float, ctypes.c_float],
            "oracle_act_rowsum": [P, I64, I64, P],
            "oracle_pack_int4": [P, I64, I64, P],
            "oracle_layernorm_quant": [P, I64, I64, P, P, ctypes.c_float, P, P, P, P, P],
            "oracle_quant_act_given_scale": [P, I64, I64, P, P, P],
            "oracle_unpack_int4": [P, I64, I64, P],
            "oracle_dequant_asym": [P, P, P, P, P, I64, I64, P, P],
            "oracle_static_ema": [ctypes.c_float, ctypes.c_float, ctypes.c_float, I],
            "oracle_quant_act_static": [P, I64, I64, P, ctypes.c_float, P],
            "oracle_to_bf16": [P, I64, P],
            "oracle_weight_codes_asym": [P, I64, I64, P, P, P],
            "oracle_pairwise_sum": [P, I64],
        }
        for name, args in sig.items():
            fn = getattr(_lib, name)
            fn.argtypes = args
            fn.restype = None
        _lib.oracle_ssz_quant_weight.restype = ctypes.c_int
        _lib.oracle_channel_mse.restype = ctypes.c_double
        _lib.oracle_static_batch_absmax.restype = ctypes.c_float
        _lib.oracle_ssz_quant_weight_asym.restype = ctypes.c_int
        _lib.oracle_channel_mse_asym.restype = ctypes.c_double
        _lib.oracle_static_ema.restype = ctypes.c_float
        _lib.oracle_pairwise_sum.restype = ctypes.c_double
    return _lib


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


# --------------------------------------------------------------------- step 1
def calib_absmax(x, ax=None) -> np.ndarray:
    """Per-input-channel absmax of x [M,K]; with ax given, the running max."""
    x = _f32(x)
    M, K = x.shape
    out = np.zeros(K, np.float32) if ax is None else _f32(ax).copy()
    _L().oracle_calib_absmax(_ptr(x), M, K, _ptr(out), 0 if ax is None else 1)
    return out


# --------------------------------------------------------------------- step 2
def weight_col_absmax(w) -> np.ndarray:
    w = _f32(w)
    N, K = w.shape
    out = np.empty(K, np.float32)
    _L().oracle_weight_col_absmax(_ptr(w), N, K, _ptr(out))
    return out


def smooth_factor(ax, aw, alpha: float):
    """s = ax^alpha / aw^(1-alpha) (fp64, rounded once), inv_s = 1/s (fp32)."""
    ax, aw = _f32(ax), _f32(aw)
    K = ax.shape[0]
    s = np.empty(K, np.float32)
    inv_s = np.empty(K, np.float32)
    _L().oracle_smooth_factor(_ptr(ax), _ptr(aw), K, float(alpha), _ptr(s), _ptr(inv_s))
    return s, inv_s


def scale_columns(a, f) -> np.ndarray:
    """a[r, j] * f[j] in fp32: the fold W' = W diag(s) or X' = X diag(1/s)."""
    a, f = _f32(a), _f32(f)
    R, K = a.shape
    out = np.empty_like(a)
    _L().oracle_scale_columns(_ptr(a), R, K, _ptr(f), _ptr(out))
    return out


# --------------------------------------------------------------------- step 3
def ssz_quant_weight(w, bits: int = 8, max_iters: int = SSZ_ITERS, s=None,
                     trace: bool = False):
    """SSZ per-output-channel symmetric quantization of w [N,K].

    With s given, w is first folded (w * s per column).  Returns a dict with
    q (int8 [N,K]), scale (fp32 [N]), mse (fp64 [N]), iters (int32 [N]) and,
    with trace=True, trace (fp64 [N, max_iters+1]).
    """
    w = _f32(w)
    if s is not None:
        w = scale_columns(w, s)
    N, K = w.shape
    q = np.empty((N, K), np.int8)
    scale = np.empty(N, np.float32)
    mse = np.empty(N, np.float64)
    iters = np.empty(N, np.int32)
    tr = np.empty((N, max_iters + 1), np.float64) if trace else None
    rc = _L().oracle_ssz_quant_weight(_ptr(w), N, K, int(bits), int(max_iters), _ptr(q),
                                      _ptr(scale), _ptr(mse), _ptr(iters), _ptr(tr))
    if rc != 0:
        raise ValueError("oracle: unsupported SSZ arguments (bits=%r, shape=%r)" % (bits, w.shape))
    out = {"q": q, "scale": scale, "mse": mse, "iters": iters}
    if trace:
        out["trace"] = tr
    return out


def weight_codes(w, scale, bits: int = 8) -> np.ndarray:
    """Codes clamp(rint(w / scale[n]), -qmax, qmax) of a folded weight."""
    w, scale = _f32(w), _f32(scale)
    N, K = w.shape
    q = np.empty((N, K), np.int8)
    _L().oracle_weight_codes(_ptr(w), N, K, int(bits), _ptr(scale), _ptr(q))
    return q


def channel_mse(w_row, scale: float, bits: int = 8) -> float:
    w_row = _f32(w_row)
    return _L().oracle_channel_mse(_ptr(w_row), w_row.shape[0], float(np.float32(scale)), int(bits))


# --------------------------------------------------------------------- step 4
def quant_act_per_token(x, inv_s=None):
    """Per-token int8 codes and scales of x [M,K] (optionally times inv_s)."""
    x = _f32(x)
    M, K = x.shape
    inv = None if inv_s is None else _f32(inv_s)
    q = np.empty((M, K), np.int8)
    sx = np.empty(M, np.float32)
    _L().oracle_quant_act_per_token(_ptr(x), M, K, _ptr(inv), _ptr(q), _ptr(sx))
    return q, sx


# ------------------------------------------------------ asymmetric int8 SSZ
def ssz_quant_weight_asym(w, max_iters: int = SSZ_ITERS, s=None, trace: bool = False):
    """Asymmetric per-channel int8 SSZ of w [N,K] (folded by s if given):
    w ~ scale * (q + 128) + offset.  Returns dict(q, scale, offset, mse,
    iters[, trace])."""
    w = _f32(w)
    if s is not None:
        w = scale_columns(w, s)
    N, K = w.shape
    q = np.empty((N, K), np.int8)
    scale = np.empty(N, np.float32)
    offset = np.empty(N, np.float32)
    mse = np.empty(N, np.float64)
    iters = np.empty(N, np.int32)
    tr = np.empty((N, max_iters + 1), np.float64) if trace else None
    rc = _L().oracle_ssz_quant_weight_asym(_ptr(w), N, K, int(max_iters), _ptr(q), _ptr(scale), _ptr(offset),
                                           _ptr(mse), _ptr(iters), _ptr(tr))
    if rc != 0:
        raise ValueError("asymmetric SSZ: unsupported arguments")
    out = dict(q=q, scale=scale, offset=offset, mse=mse, iters=iters)
    if trace:
        out["trace"] = tr
    return out


def weight_codes_asym(w, scale, offset) -> np.ndarray:
    """Stored asymmetric codes q = clamp(rint(fl(w - offset[n]) / scale[n]),
    0, 255) - 128 of a folded weight at given per-row (scale, offset)."""
    w, scale, offset = _f32(w), _f32(scale), _f32(offset)
    N, K = w.shape
    q = np.empty((N, K), np.int8)
    _L().oracle_weight_codes_asym(_ptr(w), N, K, _ptr(scale), _ptr(offset), _ptr(q))
    return q


def channel_mse_asym(w_row, S, m) -> float:
    w_row = _f32(w_row)
    return float(_L().oracle_channel_mse_asym(_ptr(w_row), w_row.shape[0], float(S), float(m)))


def quant_act_given_scale(x, inv_s, sx):
    """Codes of x [M,K] (times inv_s) at the given per-row scales sx [M]."""
    x = _f32(x)
    M, K = x.shape
    inv = None if inv_s is None else _f32(inv_s)
    sx = _f32(sx)
    q = np.empty((M, K), np.int8)
    _L().oracle_quant_act_given_scale(_ptr(x), M, K, _ptr(inv), _ptr(sx), _ptr(q))
    return q


def pairwise_sum(v) -> float:
    """The pairwise (recursive halving, zero-padded to a power of two) fp64
    sum the LayerNorm statistics use."""
    v = np.ascontiguousarray(np.asarray(v, dtype=np.float64))
    return float(_L().oracle_pairwise_sum(_ptr(v), v.shape[0]))


def layernorm_quant(h, gamma=None, beta=None, eps: float = 1e-5, inv_s=None, stats: bool = False):
    """LayerNorm (fp64 pairwise statistics, fp32 output) of h [M,K] times
    inv_s, then per-token int8 codes.  Returns (q, sx, y) with y the
    LayerNorm output, and with stats=True also [M,2] fp64 (mean, var)."""
    h = _f32(h)
    M, K = h.shape
    g = None if gamma is None else _f32(gamma)
    b = None if beta is None else _f32(beta)
    inv = None if inv_s is None else _f32(inv_s)
    q = np.empty((M, K), np.int8)
    sx = np.empty(M, np.float32)
    y = np.empty((M, K), np.float32)
    st = np.empty((M, 2), np.float64) if stats else None
    _L().oracle_layernorm_quant(_ptr(h), M, K, _ptr(g), _ptr(b), float(eps), _ptr(inv), _ptr(q), _ptr(sx), _ptr(y),
                                _ptr(st))
    return (q, sx, y, st) if stats else (q, sx, y)


def pack_int4(q) -> np.ndarray:
    """Two int4 codes per byte: element 2i low nibble, 2i+1 high nibble."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    N, K = q.shape
    out = np.empty((N, K // 2), np.uint8)
    _L().oracle_pack_int4(_ptr(q), N, K, _ptr(out))
    return out


def unpack_int4(packed, K: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    N = packed.shape[0]
    out = np.empty((N, K), np.int8)
    _L().oracle_unpack_int4(_ptr(packed), N, K, _ptr(out))
    return out


def act_rowsum(qx) -> np.ndarray:
    qx = np.ascontiguousarray(qx, dtype=np.int8)
    M, K = qx.shape
    R = np.empty(M, np.int32)
    _L().oracle_act_rowsum(_ptr(qx), M, K, _ptr(R))
    return R


def dequant_asym(acc, R, sx, S, m, out: str = "bf16") -> np.ndarray:
    """sx (S (acc + 128 R) + m R) in fp32; out as in dequant."""
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    R = np.ascontiguousarray(R, dtype=np.int32)
    sx, S, m = _f32(sx), _f32(S), _f32(m)
    M, N = acc.shape
    if out == "f32":
        y = np.empty((M, N), np.float32)
        _L().oracle_dequant_asym(_ptr(acc), _ptr(R), _ptr(sx), _ptr(S), _ptr(m), M, N, _ptr(y), None)
    else:
        y = np.empty((M, N), np.uint16)
        _L().oracle_dequant_asym(_ptr(acc), _ptr(R), _ptr(sx), _ptr(S), _ptr(m), M, N, None, _ptr(y))
    return y


# ------------------------------------------------------ static activation scale
STATIC_EMA_RATE = np.float32(0.9)


def static_batch_absmax(x, inv_s=None) -> np.float32:
    """max |x * inv_s| over one calibration batch x [M,K]."""
    x = _f32(x)
    M, K = x.shape
    inv = None if inv_s is None else _f32(inv_s)
    return np.float32(_L().oracle_static_batch_absmax(_ptr(x), M, K, _ptr(inv)))


def static_ema(state, a, rate=STATIC_EMA_RATE, first=False) -> np.float32:
    """One moving-average step of the per-tensor activation range (fp32)."""
    return np.float32(_L().oracle_static_ema(float(state), float(a), float(rate), 1 if first else 0))


def static_range(batches, inv_s=None, rate=STATIC_EMA_RATE) -> np.float32:
    """Moving-average abs-max over a sequence of calibration batches."""
    m = np.float32(0.0)
    for i, xb in enumerate(batches):
        m = static_ema(m, static_batch_absmax(xb, inv_s), rate, first=(i == 0))
    return m


def quant_act_static(x, inv_s, m):
    """Codes of x [M,K] (times inv_s) at the static scale S = m / 127."""
    x = _f32(x)
    M, K = x.shape
    inv = None if inv_s is None else _f32(inv_s)
    q = np.empty((M, K), np.int8)
    _L().oracle_quant_act_static(_ptr(x), M, K, _ptr(inv), float(np.float32(m)), _ptr(q))
    return q


def static_scale(m) -> np.float32:
    """S = m / 127 in fp32."""
    return np.float32(np.float32(m) / np.float32(127.0))


# --------------------------------------------------------------------- step 5
def gemm_i8(qx, qw) -> np.ndarray:
    """Exact int32 acc[t,n] = sum_k qx[t,k] * qw[n,k]."""
    qx = np.ascontiguousarray(qx, dtype=np.int8)
    qw = np.ascontiguousarray(qw, dtype=np.int8)
    M, K = qx.shape
    N, K2 = qw.shape
    assert K == K2
    acc = np.empty((M, N), np.int32)
    _L().oracle_gemm_i8(_ptr(qx), _ptr(qw), M, N, K, _ptr(acc))
    return acc


def dequant(acc, sx, sw, out: str = "bf16") -> np.ndarray:
    """((float)acc * sx[t]) * sw[n]; out='f32' gives fp32, 'bf16' the RNE bf16
    bit patterns as uint16."""
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    sx, sw = _f32(sx), _f32(sw)
    M, N = acc.shape
    if out == "f32":
        y = np.empty((M, N), np.float32)
        _L().oracle_dequant(_ptr(acc), _ptr(sx), _ptr(sw), M, N, _ptr(y), None)
    else:
        y = np.empty((M, N), np.uint16)
        _L().oracle_dequant(_ptr(acc), _ptr(sx), _ptr(sw), M, N, None, _ptr(y))
    return y


def to_bf16_bits(a) -> np.ndarray:
    a = _f32(a)
    out = np.empty(a.shape, np.uint16)
    _L().oracle_to_bf16(_ptr(a), a.size, _ptr(out))
    return out


def bf16_bits_to_f32(b) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


# ----------------------------------------------------------------- whole path
def linear(x, w, alpha: float, bits: int = 8, max_iters: int = SSZ_ITERS,
           out: str = "bf16", ax=None):
    """The whole path from raw inputs: calibrate on x (or use ax), smooth,
    SSZ-quantize the folded weight, quantize the folded activations per token,
    integer product and dequant.  Returns every intermediate."""
    x, w = _f32(x), _f32(w)
    ax = calib_absmax(x) if ax is None else _f32(ax)
    aw = weight_col_absmax(w)
    s, inv_s = smooth_factor(ax, aw, alpha)
    wq = ssz_quant_weight(w, bits, max_iters, s=s)
    qx, sx = quant_act_per_token(x, inv_s)
    acc = gemm_i8(qx, wq["q"])
    y = dequant(acc, sx, wq["scale"], out=out)
    return {"ax": ax, "aw": aw, "s": s, "inv_s": inv_s, "qw": wq["q"], "sw": wq["scale"],
            "mse": wq["mse"], "iters": wq["iters"], "qx": qx, "sx": sx, "acc": acc, "y": y}
