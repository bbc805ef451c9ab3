"""The debug build's counters (sq_debug_status): non-finite inputs and
failed index checks, counted on the device, read and cleared on the host.

The pages' debugging advice (CUDA INT8 notes section 5: copy the parameters
back and compare stage by stage) in place of a sanitizer.  The debug build is
a second library (libw8a8_debug.so, the same kernels compiled with
-DW8A8_DEBUG) loaded here beside the release one.  Nothing here faults or
traps: non-finite inputs are valid data the kernels process like any other.
"""
import ctypes
import os

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int


@pytest.fixture(scope="module")
def dbg():
    import importlib.util
    spec = importlib.util.spec_from_file_location("w8a8_build", os.path.join(ROOT, "w8a8_linear_layers_b200",
                                                                             "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    lib = ctypes.CDLL(b.build(debug=True))
    lib.sq_debug_status.argtypes = [P, P, P, P]
    lib.quant_act_per_token.argtypes = [P, I, I64, I64, P, P, P, P]
    lib.sq_calib_absmax.argtypes = [P, I, I64, I64, P, I, P]
    lib.ssz_quant_weight.argtypes = [P, I, I64, I64, P, I, I, P, P, P, P, P]
    return lib


def _status(lib):
    nf, ix, en = ctypes.c_uint64(), ctypes.c_uint64(), ctypes.c_int()
    assert lib.sq_debug_status(None, ctypes.byref(nf), ctypes.byref(ix), ctypes.byref(en)) == 0
    return nf.value, ix.value, en.value


def test_release_build_reports_disabled():
    import w8a8_linear_layers_b200 as w
    assert w.debug_status() == (0, 0, False)


def test_debug_build_counts_nonfinite_inputs(dbg):
    _status(dbg)  # clear
    M, K = 37, 1040
    x = torch.randn(M, K, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    x[0, 5] = float("inf")
    x[4, 1039] = float("-inf")
    x[36, 0] = float("nan")
    xd = x.cuda()
    q = torch.empty(M, K, dtype=torch.int8, device="cuda")
    sx = torch.empty(M, device="cuda")
    assert dbg.quant_act_per_token(xd.data_ptr(), 1, M, K, None, q.data_ptr(), sx.data_ptr(), None) == 0
    assert _status(dbg) == (3, 0, 1)
    assert _status(dbg) == (0, 0, 1)  # read and cleared
    ax = torch.empty(K, device="cuda")
    assert dbg.sq_calib_absmax(xd.data_ptr(), 1, M, K, ax.data_ptr(), 0, None) == 0
    assert _status(dbg) == (3, 0, 1)
    # weights: the search counts the non-finite (smoothed) weights it reads
    wt = torch.randn(64, 512, generator=torch.Generator().manual_seed(4)) * 0.02
    wt[7, 100] = float("inf")
    wd = wt.cuda()
    qw = torch.empty(64, 512, dtype=torch.int8, device="cuda")
    sw = torch.empty(64, device="cuda")
    assert dbg.ssz_quant_weight(wd.data_ptr(), 0, 64, 512, None, 8, 20, qw.data_ptr(), sw.data_ptr(), None, None,
                                None) == 0
    assert _status(dbg) == (1, 0, 1)


def test_debug_build_computes_what_the_release_build_does(dbg):
    """Finite inputs: no counts, and the same codes and scales as the release
    library."""
    import w8a8_linear_layers_b200 as w
    _status(dbg)
    M, K = 300, 4096
    x = (torch.randn(M, K, generator=torch.Generator().manual_seed(5)) * 3).to(torch.bfloat16).cuda()
    inv = torch.rand(K, generator=torch.Generator().manual_seed(6)).cuda() + 0.5
    q1, q2 = (torch.empty(M, K, dtype=torch.int8, device="cuda") for _ in range(2))
    s1, s2 = (torch.empty(M, device="cuda") for _ in range(2))
    w.quant_act_per_token(x, inv, q1, s1)
    assert dbg.quant_act_per_token(x.data_ptr(), 1, M, K, inv.data_ptr(), q2.data_ptr(), s2.data_ptr(), None) == 0
    torch.cuda.synchronize()
    assert torch.equal(q1, q2) and torch.equal(s1, s2)
    assert _status(dbg) == (0, 0, 1)
