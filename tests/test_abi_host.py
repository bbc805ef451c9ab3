"""Host-side checks of the C ABI (no GPU needed).

The library must load, export every function include/w8a8.h declares, and
reject bad arguments on the host -- before any device work -- with the
documented status codes.  Pointers here are fake addresses: validation never
dereferences them, and no call reaches a kernel launch.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "w8a8.h")


@pytest.fixture(scope="module")
def lib():
    from tests.conftest import build_cuda_library
    build_cuda_library()
    import w8a8_linear_layers_b200 as w
    return w.lib


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sq_\w+|ssz_\w+|quant_\w+|w8a8_\w+|w4a8_\w+)\s*\(", text)))


def test_header_declares_the_five_steps():
    fns = declared_functions()
    for name in ["sq_calib_absmax", "sq_smooth_fold", "ssz_quant_weight", "quant_act_per_token",
                 "w8a8_gemm_dequant"]:
        assert name in fns


def test_library_exports_every_declared_symbol(lib):
    import w8a8_linear_layers_b200 as w
    fns = declared_functions()
    missing = [f for f in fns if not hasattr(lib, f)]
    assert missing == []
    assert sorted(w.EXPORTS) == sorted(fns)


def test_status_strings_and_version(lib):
    assert lib.sq_abi_version() == 1
    names = [lib.sq_status_string(i).decode() for i in range(9)]
    assert names == ["SQ_OK", "SQ_ERR_NULL", "SQ_ERR_SHAPE", "SQ_ERR_DTYPE", "SQ_ERR_ALIGN", "SQ_ERR_ARG",
                     "SQ_ERR_UNSUPPORTED", "SQ_ERR_CUDA", "SQ_ERR_DEVICE"]
    assert lib.sq_status_string(99).decode() == "SQ_ERR_UNKNOWN"


A = 0x7f0000000000  # a fake, 256-byte aligned device address (never dereferenced)


def P(off=0):
    return ctypes.c_void_p(A + off)


NULL = None


def _detail(lib):
    return lib.sq_last_error_detail().decode()


@pytest.mark.parametrize("case,status", [
    ("null_x", 1), ("null_absmax", 1), ("bad_dtype", 3), ("k_not_16", 2), ("k_zero", 2), ("neg_m", 2),
    ("misaligned_x", 4),
])
def test_calib_absmax_rejects(lib, case, status):
    args = dict(x=P(), xt=1, M=4, K=32, ax=P(4096), acc=0)
    if case == "null_x": args["x"] = NULL
    if case == "null_absmax": args["ax"] = NULL
    if case == "bad_dtype": args["xt"] = 7
    if case == "k_not_16": args["K"] = 40
    if case == "k_zero": args["K"] = 0
    if case == "neg_m": args["M"] = -1
    if case == "misaligned_x": args["x"] = P(2)
    rc = lib.sq_calib_absmax(args["x"], args["xt"], args["M"], args["K"], args["ax"], args["acc"], None)
    assert rc == status, _detail(lib)
    assert _detail(lib).startswith("sq_calib_absmax")


@pytest.mark.parametrize("alpha,status", [(-0.1, 5), (1.5, 5), (float("nan"), 5)])
def test_smooth_fold_rejects_alpha(lib, alpha, status):
    rc = lib.sq_smooth_fold(P(), P(4096), 1, 8, 32, alpha, P(8192), P(12288), P(16384), NULL, None)
    assert rc == status
    assert "alpha" in _detail(lib)


def test_smooth_fold_fold_needs_16_byte_s(lib):
    # s_out at a 4-byte offset is a valid vector, but the materialised fold
    # reads it 16 bytes at a time
    rc = lib.sq_smooth_fold(P(), P(4096), 1, 8, 32, 0.5, P(8192), P(12292), P(16384), P(32768), None)
    assert rc == 4, _detail(lib)
    assert "s_out" in _detail(lib)


def test_smooth_factor_rejects(lib):
    assert lib.sq_smooth_factor(NULL, P(4096), 32, 0.5, P(8192), P(12288), None) == 1
    assert lib.sq_smooth_factor(P(), P(4096), 40, 0.5, P(8192), P(12288), None) == 2
    assert lib.sq_smooth_factor(P(), P(4096), 0, 0.5, P(8192), P(12288), None) == 2
    assert lib.sq_smooth_factor(P(), P(4096), 32, 1.5, P(8192), P(12288), None) == 5
    assert "alpha" in _detail(lib)
    assert lib.sq_smooth_factor(P(), P(4098), 32, 0.5, P(8192), P(12288), None) == 4


@pytest.mark.parametrize("case,status", [
    ("bits6", 5), ("iters_neg", 5), ("iters_big", 5), ("k_big", 2), ("k_odd", 2), ("null_q", 1),
    ("misaligned_s", 4), ("dtype", 3),
])
def test_ssz_rejects(lib, case, status):
    a = dict(w=P(), wt=1, N=8, K=64, s=P(4096), bits=8, it=20, q=P(8192), sc=P(12288), mse=NULL, its=NULL)
    if case == "bits6": a["bits"] = 6
    if case == "iters_neg": a["it"] = -1
    if case == "iters_big": a["it"] = 256
    if case == "k_big": a["K"] = 32784
    if case == "k_odd": a["K"] = 72
    if case == "null_q": a["q"] = NULL
    if case == "misaligned_s": a["s"] = P(4)
    if case == "dtype": a["wt"] = 2
    rc = lib.ssz_quant_weight(a["w"], a["wt"], a["N"], a["K"], a["s"], a["bits"], a["it"], a["q"], a["sc"],
                              a["mse"], a["its"], None)
    assert rc == status, _detail(lib)


@pytest.mark.parametrize("case,status", [("null", 1), ("k", 2), ("align_q", 4), ("dtype", 3)])
def test_quant_act_rejects(lib, case, status):
    a = dict(x=P(), xt=1, M=4, K=64, inv=NULL, q=P(8192), sc=P(12288))
    if case == "null": a["q"] = NULL
    if case == "k": a["K"] = 65
    if case == "align_q": a["q"] = P(8)
    if case == "dtype": a["xt"] = 5
    rc = lib.quant_act_per_token(a["x"], a["xt"], a["M"], a["K"], a["inv"], a["q"], a["sc"], None)
    assert rc == status, _detail(lib)


@pytest.mark.parametrize("case,status", [("null_off", 1), ("k", 2), ("iters", 5), ("align_off", 4), ("dtype", 3)])
def test_ssz_asym_rejects(lib, case, status):
    a = dict(w=P(), wt=1, N=4, K=64, s=NULL, it=20, q=P(8192), sc=P(12288), off=P(12544))
    if case == "null_off": a["off"] = NULL
    if case == "k": a["K"] = 40
    if case == "iters": a["it"] = 300
    if case == "align_off": a["off"] = P(2)
    if case == "dtype": a["wt"] = 4
    rc = lib.ssz_quant_weight_asym(a["w"], a["wt"], a["N"], a["K"], a["s"], a["it"], a["q"], a["sc"], a["off"],
                                   NULL, NULL, None)
    assert rc == status, _detail(lib)


@pytest.mark.parametrize("case,status", [("null_rs", 1), ("null_ow", 1), ("k_asym_limit", 2), ("align_ow", 4)])
def test_gemm_asym_rejects(lib, case, status):
    a = dict(qx=P(), sx=P(4096), rs=P(4608), qw=P(8192), sw=P(12288), ow=P(12544), M=4, N=16, K=64, y=P(16384))
    if case == "null_rs": a["rs"] = NULL
    if case == "null_ow": a["ow"] = NULL
    if case == "k_asym_limit": a["K"] = 65808
    if case == "align_ow": a["ow"] = P(12548)
    rc = lib.w8a8_gemm_dequant_asym(a["qx"], a["sx"], a["rs"], a["qw"], a["sw"], a["ow"], a["M"], a["N"], a["K"],
                                    a["y"], 1, NULL, None)
    assert rc == status, _detail(lib)


@pytest.mark.parametrize("case,status", [("null", 1), ("k16", 2), ("k_limit", 2), ("align", 4), ("dtype", 3)])
def test_w4a8_rejects(lib, case, status):
    a = dict(qx=P(), sx=P(4096), qw=P(8192), sw=P(12288), M=4, N=16, K=64, y=P(16384), yt=1)
    if case == "null": a["qw"] = NULL
    if case == "k16": a["K"] = 48
    if case == "k_limit": a["K"] = 131072  # 16 * 128 * 8 * K would pass 2^31
    if case == "align": a["qw"] = P(8200)
    if case == "dtype": a["yt"] = 2
    rc = lib.w4a8_gemm_dequant(a["qx"], a["sx"], a["qw"], a["sw"], a["M"], a["N"], a["K"], a["y"], a["yt"], NULL,
                               None)
    assert rc == status, _detail(lib)
    assert lib.sq_pack_int4(P(), 4, 48, P(4096), None) == 2
    assert lib.sq_pack_int4(P(), 4, 64, NULL, None) == 1


@pytest.mark.parametrize("case,status", [("null", 1), ("k", 2), ("k_big", 2), ("eps", 5), ("align_g", 4),
                                         ("dtype", 3)])
def test_layernorm_quant_rejects(lib, case, status):
    a = dict(h=P(), ht=1, M=4, K=64, g=NULL, b=NULL, eps=1e-5, inv=NULL, q=P(8192), sc=P(12288))
    if case == "null": a["sc"] = NULL
    if case == "k": a["K"] = 40
    if case == "k_big": a["K"] = 16400
    if case == "eps": a["eps"] = -1.0
    if case == "align_g": a["g"] = P(4)
    if case == "dtype": a["ht"] = 6
    rc = lib.sq_layernorm_quant(a["h"], a["ht"], a["M"], a["K"], a["g"], a["b"], a["eps"], a["inv"], a["q"], a["sc"],
                                None)
    assert rc == status, _detail(lib)


def test_sharded_helpers_reject(lib):
    assert lib.quant_act_given_scale(P(), 1, 4, 64, NULL, NULL, P(8192), None) == 1
    assert lib.quant_act_given_scale(P(), 1, 4, 40, NULL, P(4096), P(8192), None) == 2
    assert lib.quant_act_given_scale(P(), 1, 4, 64, NULL, P(4096), P(8200), None) == 4
    assert lib.quant_act_given_scale(NULL, 1, 0, 64, NULL, NULL, NULL, None) == 0
    assert lib.sq_dequant(P(), P(4096), P(8192), 4, 16, NULL, 1, None) == 1
    assert lib.sq_dequant(P(), P(4096), P(8192), 4, 18, P(12288), 1, None) == 2
    assert lib.sq_dequant(P(4), P(4096), P(8192), 4, 16, P(12288), 1, None) == 4
    assert lib.sq_dequant(P(), P(4096), P(8192), 4, 16, P(12288), 7, None) == 3


def test_quant_rowsum_rejects_misaligned(lib):
    assert lib.quant_act_per_token_rowsum(P(), 1, 4, 64, NULL, P(8192), P(12288), P(2), None) == 4


@pytest.mark.parametrize("case,status", [("null", 1), ("null_range", 1), ("k", 2), ("align_q", 4),
                                         ("dtype", 3)])
def test_quant_act_static_rejects(lib, case, status):
    a = dict(x=P(), xt=1, M=4, K=64, inv=NULL, rng=P(4096), q=P(8192), sc=NULL)
    if case == "null": a["q"] = NULL
    if case == "null_range": a["rng"] = NULL
    if case == "k": a["K"] = 65
    if case == "align_q": a["q"] = P(8)
    if case == "dtype": a["xt"] = 5
    rc = lib.quant_act_static(a["x"], a["xt"], a["M"], a["K"], a["inv"], a["rng"], a["q"], a["sc"], NULL, None)
    assert rc == status, _detail(lib)


@pytest.mark.parametrize("case,status", [("null", 1), ("k", 2), ("rate_neg", 5), ("rate_big", 5),
                                         ("rate_nan", 5), ("align", 4)])
def test_static_range_update_rejects(lib, case, status):
    a = dict(ax=P(), inv=NULL, K=64, rate=0.9, rng=P(4096))
    if case == "null": a["rng"] = NULL
    if case == "k": a["K"] = 0
    if case == "rate_neg": a["rate"] = -0.1
    if case == "rate_big": a["rate"] = 1.5
    if case == "rate_nan": a["rate"] = float("nan")
    if case == "align": a["ax"] = P(2)
    rc = lib.sq_static_range_update(a["ax"], a["inv"], a["K"], a["rate"], 0, a["rng"], None)
    assert rc == status, _detail(lib)


@pytest.mark.parametrize("case,status", [
    ("null_sw", 1), ("k", 2), ("n_bf16", 2), ("n_f32", 2), ("align_y", 4), ("dtype", 3), ("k_huge", 2),
])
def test_gemm_rejects(lib, case, status):
    a = dict(qx=P(), sx=P(4096), qw=P(8192), sw=P(12288), M=4, N=16, K=64, y=P(16384), yt=1, acc=NULL)
    if case == "null_sw": a["sw"] = NULL
    if case == "k": a["K"] = 24
    if case == "n_bf16": a["N"] = 12
    if case == "n_f32": a.update(N=10, yt=0)
    if case == "align_y": a["y"] = P(8)
    if case == "dtype": a["yt"] = 3
    if case == "k_huge": a["K"] = 133152
    rc = lib.w8a8_gemm_dequant(a["qx"], a["sx"], a["qw"], a["sw"], a["M"], a["N"], a["K"], a["y"], a["yt"],
                               a["acc"], None)
    assert rc == status, _detail(lib)


def test_empty_inputs_are_noops(lib):
    # M == 0 / N == 0 return OK without touching the device
    assert lib.quant_act_per_token(NULL, 1, 0, 64, NULL, NULL, NULL, None) == 0
    assert lib.quant_act_static(NULL, 1, 0, 64, NULL, NULL, NULL, NULL, NULL, None) == 0
    assert lib.ssz_quant_weight(NULL, 1, 0, 64, NULL, 8, 20, NULL, NULL, NULL, NULL, None) == 0
    assert lib.w8a8_gemm_dequant(NULL, NULL, NULL, NULL, 0, 16, 64, NULL, 1, NULL, None) == 0
    assert lib.w8a8_gemm_dequant(NULL, NULL, NULL, NULL, 4, 0, 64, NULL, 1, NULL, None) == 0


def test_python_binding_refuses_cpu_tensors():
    import torch
    import w8a8_linear_layers_b200 as w
    x = torch.zeros(4, 32, dtype=torch.bfloat16)
    ax = torch.zeros(32)
    with pytest.raises(ValueError):
        w.sq_calib_absmax(x, ax)


def test_debug_status_release_build(lib):
    nf, ix, en = ctypes.c_uint64(7), ctypes.c_uint64(7), ctypes.c_int(7)
    assert lib.sq_debug_status(None, ctypes.byref(nf), ctypes.byref(ix), ctypes.byref(en)) == 0
    assert (nf.value, ix.value, en.value) == (0, 0, 0)
    assert lib.sq_debug_status(None, None, ctypes.byref(ix), ctypes.byref(en)) == 1


def test_debug_library_exports_every_declared_symbol():
    """The debug build (-DW8A8_DEBUG) is the same library with counters: it
    exports every declared entry point."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("w8a8_build", os.path.join(ROOT, "w8a8_linear_layers_b200",
                                                                             "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    dbg = ctypes.CDLL(b.build(debug=True))
    assert [f for f in declared_functions() if not hasattr(dbg, f)] == []
