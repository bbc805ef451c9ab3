"""Pins of the CPU oracle against things other than itself.

Each test checks the oracle against what the pages and mathematics fix:
library routines (numpy/torch), closed forms, invariants, hand-derived golden
values under tests/golden/, and brute force on tiny inputs.  They are chosen so
that a plausible slip (a dropped term, a wrong sign or index, a transposed
operand, a swapped exponent) fails at least one; tests/test_oracle_mutants.py
plants such slips in a copy of the oracle and checks that they are caught.

Sources: SmoothQuant deep-dive (developer.baidu.com) section 1 for the
smoothing factor and the equivalence; "SSZ：权重量化算法说明" (msModelSlim)
sections 算法流程 / 迭代优化阶段 / 收敛判断 / 算法参数 for the weight search;
CUDA INT8 notes (aicoding.csdn.net) section 2.1 for Q = round(R/S) + Z;
"PaddleNLP GPT 量化感知训练（QAT）实战指南" section 六 for the moving-average
activation range.
"""
import math
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


def _llm_like(M, K, n_out=2, scale=40.0, seed=0):
    r = np.random.default_rng(seed)
    x = r.standard_normal((M, K)).astype(np.float32)
    cols = r.permutation(K)[:n_out]
    x[:, cols] *= scale
    return x


# ----------------------------------------------------------------- step 1 / 2a
def test_calib_absmax_matches_numpy(orc):
    x = _llm_like(37, 80)
    np.testing.assert_array_equal(orc.calib_absmax(x), np.abs(x).max(axis=0))


def test_calib_absmax_running_max_equals_concatenation(orc):
    x1, x2 = _llm_like(9, 48, seed=1), _llm_like(13, 48, seed=2)
    run = orc.calib_absmax(x2, ax=orc.calib_absmax(x1))
    np.testing.assert_array_equal(run, orc.calib_absmax(np.concatenate([x1, x2])))
    # a larger prior max survives
    big = np.full(48, 1e6, np.float32)
    np.testing.assert_array_equal(orc.calib_absmax(x1, ax=big), big)


def test_weight_col_absmax_is_per_input_channel(orc):
    w = rng.standard_normal((11, 24)).astype(np.float32)
    np.testing.assert_array_equal(orc.weight_col_absmax(w), np.abs(w).max(axis=0))
    # column (input channel) reduction, not row: a planted column max shows up at j
    w[3, 5] = 100.0
    assert orc.weight_col_absmax(w)[5] == 100.0


# ----------------------------------------------------------------- step 2
def _ax_aw(K=64, seed=3):
    r = np.random.default_rng(seed)
    ax = (np.abs(r.standard_normal(K)) * 5 + 0.1).astype(np.float32)
    aw = (np.abs(r.standard_normal(K)) * 0.05 + 0.01).astype(np.float32)
    return ax, aw


def test_smooth_factor_special_alphas(orc):
    ax, aw = _ax_aw()
    s1, inv1 = orc.smooth_factor(ax, aw, 1.0)           # alpha = 1: s = max|X_j|
    np.testing.assert_array_equal(s1, ax)
    s0, _ = orc.smooth_factor(ax, aw, 0.0)              # alpha = 0: s = 1 / max|W_j|
    np.testing.assert_array_equal(s0, (1.0 / aw.astype(np.float64)).astype(np.float32))
    sh, _ = orc.smooth_factor(ax, aw, 0.5)              # alpha = 1/2: sqrt(ax / aw)
    np.testing.assert_allclose(sh, np.sqrt(ax.astype(np.float64) / aw), rtol=2e-7)
    np.testing.assert_array_equal(inv1, np.float32(1.0) / s1)


def test_smooth_factor_matches_torch_pow(orc):
    ax, aw = _ax_aw(K=128, seed=4)
    for alpha in (0.2, 0.5, 0.8):
        s, _ = orc.smooth_factor(ax, aw, alpha)
        a = torch.tensor(ax, dtype=torch.float64)
        b = torch.tensor(aw, dtype=torch.float64)
        ref = (a.pow(float(np.float32(alpha))) / b.pow(1.0 - float(np.float32(alpha)))).float().numpy()
        np.testing.assert_allclose(s, ref, rtol=1.2e-7)


def test_smooth_factor_zero_channel_is_identity(orc):
    ax, aw = _ax_aw(K=8)
    ax[2] = 0.0
    aw[5] = 0.0
    s, inv = orc.smooth_factor(ax, aw, 0.5)
    assert s[2] == 1.0 and inv[2] == 1.0 and s[5] == 1.0


def test_smoothing_balances_ranges(orc):
    # alpha = 1/2: after the fold, max|X'_j| and max|W'_j| both equal
    # sqrt(max|X_j| * max|W_j|)  (the "balance" the page describes)
    x = _llm_like(64, 96, n_out=4, scale=50.0, seed=5)
    w = (np.random.default_rng(6).standard_normal((40, 96)) * 0.02).astype(np.float32)
    ax, aw = orc.calib_absmax(x), orc.weight_col_absmax(w)
    s, inv_s = orc.smooth_factor(ax, aw, 0.5)
    xs, ws = orc.scale_columns(x, inv_s), orc.scale_columns(w, s)
    target = np.sqrt(ax.astype(np.float64) * aw)
    np.testing.assert_allclose(np.abs(xs).max(0), target, rtol=4e-7)
    np.testing.assert_allclose(np.abs(ws).max(0), target, rtol=4e-7)
    # alpha = 1 makes every activation channel range 1; alpha = 0 every weight column range 1
    s1, inv1 = orc.smooth_factor(ax, aw, 1.0)
    np.testing.assert_allclose(np.abs(orc.scale_columns(x, inv1)).max(0), 1.0, rtol=1.2e-7)
    s0, _ = orc.smooth_factor(ax, aw, 0.0)
    np.testing.assert_allclose(np.abs(orc.scale_columns(w, s0)).max(0), 1.0, rtol=1.2e-7)


def test_smoothing_is_equivalent_transform(orc):
    # (X diag(s)^-1)(W diag(s))^T = X W^T, up to the fp32 rounding of the fold
    x = _llm_like(32, 128, n_out=3, scale=60.0, seed=7)
    w = (np.random.default_rng(8).standard_normal((48, 128)) * 0.02).astype(np.float32)
    for alpha in (0.0, 0.5, 0.8, 1.0):
        s, inv_s = orc.smooth_factor(orc.calib_absmax(x), orc.weight_col_absmax(w), alpha)
        lhs = orc.scale_columns(x, inv_s).astype(np.float64) @ orc.scale_columns(w, s).astype(np.float64).T
        rhs = x.astype(np.float64) @ w.astype(np.float64).T
        # each product term carries at most ~3 fp32 roundings
        bound = 4e-7 * (np.abs(x).astype(np.float64) @ np.abs(w).astype(np.float64).T)
        assert np.all(np.abs(lhs - rhs) <= bound + 1e-30)


def test_scale_columns_matches_numpy(orc):
    a = rng.standard_normal((7, 33)).astype(np.float32)
    f = rng.standard_normal(33).astype(np.float32)
    np.testing.assert_array_equal(orc.scale_columns(a, f), a * f[None, :])


# ----------------------------------------------------------------- step 3: SSZ
def _q(w, s, qmax):
    return np.clip(np.rint(np.float32(w) / np.float32(s)), -qmax, qmax)


def _mse_np(w, s, qmax):
    q = _q(w, s, qmax).astype(np.float64)
    return float(np.mean((w.astype(np.float64) - np.float64(np.float32(s)) * q) ** 2))


def test_ssz_golden_hand_cases(orc):
    # see tests/golden/ssz_hand.txt for the derivations
    w = np.array([[1.0, 0.3]], np.float32)
    r = orc.ssz_quant_weight(w, bits=4)
    w2 = np.float64(np.float32(0.3))
    assert r["scale"][0] == np.float32((7.0 + 2.0 * w2) / 53.0)
    assert r["q"].tolist() == [[7, 2]] and r["iters"][0] == 2

    c = np.float32(2.0 ** -6)
    k = np.random.default_rng(9).integers(-127, 128, size=64).astype(np.float32)
    k[10] = 127
    r = orc.ssz_quant_weight((c * k)[None, :], bits=8)
    assert r["scale"][0] == c and r["mse"][0] == 0.0 and r["iters"][0] == 1
    np.testing.assert_array_equal(r["q"][0], k.astype(np.int8))

    row = np.zeros((1, 32), np.float32)
    row[0, 17] = 0.7
    r = orc.ssz_quant_weight(row, bits=8)
    s0 = np.float32(np.float32(0.7) / np.float32(127))
    assert r["scale"][0] == s0
    assert r["q"][0, 17] == 127 and r["iters"][0] == 1
    assert r["mse"][0] == pytest.approx((float(np.float32(0.7)) - 127.0 * float(s0)) ** 2 / 32, rel=1e-12)
    assert np.count_nonzero(r["q"]) == 1

    r = orc.ssz_quant_weight(np.zeros((1, 16), np.float32), bits=8)
    assert r["scale"][0] == np.float32(1e-5) and not r["q"].any() and r["iters"][0] == 1

    tiny = np.full((1, 16), 1e-7, np.float32)
    r = orc.ssz_quant_weight(tiny, bits=8)
    assert r["scale"][0] == np.float32(1e-5) and not r["q"].any() and r["iters"][0] == 1
    assert r["mse"][0] == pytest.approx(float(np.float32(1e-7)) ** 2, rel=1e-12)


@pytest.mark.parametrize("bits", [8, 4])
def test_ssz_never_worse_than_minmax_and_monotone(orc, bits):
    w = (np.random.default_rng(10).standard_normal((64, 256)) * 0.02).astype(np.float32)
    w[np.random.default_rng(11).random(w.shape) < 0.003] *= 10.0
    qmax = (1 << (bits - 1)) - 1
    r = orc.ssz_quant_weight(w, bits=bits, trace=True)
    tr = r["trace"]
    assert np.all(np.diff(tr, axis=1) <= 0.0)                 # greedy: never increases
    mm = orc.ssz_quant_weight(w, bits=bits, max_iters=0)
    assert np.all(mm["iters"] == 0)
    np.testing.assert_array_equal(mm["scale"], np.maximum(np.abs(w).max(1) / np.float32(qmax), np.float32(1e-5)))
    assert np.all(r["mse"] <= mm["mse"])
    # the search does real work: strictly better on most channels
    assert np.mean(r["mse"] < mm["mse"]) > 0.8
    np.testing.assert_array_equal(tr[:, 0], mm["mse"])


@pytest.mark.parametrize("bits", [8, 4])
def test_ssz_reported_error_and_codes_are_consistent(orc, bits):
    w = (np.random.default_rng(12).standard_normal((16, 64)) * 0.02).astype(np.float32)
    qmax = (1 << (bits - 1)) - 1
    r = orc.ssz_quant_weight(w, bits=bits)
    for n in range(w.shape[0]):
        np.testing.assert_array_equal(r["q"][n], _q(w[n], r["scale"][n], qmax).astype(np.int8))
        assert r["mse"][n] == pytest.approx(_mse_np(w[n], r["scale"][n], qmax), rel=1e-12)
    assert np.abs(r["q"]).max() <= qmax
    np.testing.assert_array_equal(orc.weight_codes(w, r["scale"], bits), r["q"])


@pytest.mark.parametrize("bits", [8, 4])
def test_ssz_scale_is_least_squares_for_its_codes(orc, bits):
    # closed form: for fixed codes q the residual sum (w - s q)^2 is minimised
    # at s* = sum(w q) / sum(q q); a converged channel sits at (or within a
    # rounding of) s* of its own codes, so s +/- 1% is never better.
    w = (np.random.default_rng(13).standard_normal((48, 128)) * 0.02).astype(np.float32)
    r = orc.ssz_quant_weight(w, bits=bits)
    conv = r["iters"] < 20
    assert conv.mean() > 0.9
    for n in np.nonzero(conv)[0]:
        q = r["q"][n].astype(np.float64)
        wd = w[n].astype(np.float64)
        s = float(r["scale"][n])
        s_star = (wd @ q) / (q @ q)
        assert abs(s - s_star) <= 2e-3 * s_star
        res = lambda t: float(np.sum((wd - t * q) ** 2))
        assert res(s) <= res(s * 1.01) and res(s) <= res(s * 0.99)


def test_ssz_close_to_brute_force_optimum(orc):
    # brute force on tiny rows: a dense grid of scales in [0.25, 1.5] x MinMax.
    # The search is local, so it may stop above the global optimum, but it can
    # never go below it, never ends above MinMax, and closes much of the gap.
    r8 = np.random.default_rng(14)
    for bits in (8, 4):
        qmax = (1 << (bits - 1)) - 1
        gs, gm = [], []
        for K in (24, 64):
            w = (r8.standard_normal((20, K)) * 0.02).astype(np.float32)
            r = orc.ssz_quant_weight(w, bits=bits)
            for n in range(w.shape[0]):
                s0 = np.abs(w[n]).max() / qmax
                grid = (np.linspace(0.25, 1.5, 100001) * s0).astype(np.float32)
                wd = w[n].astype(np.float64)[None, :]
                q = np.clip(np.rint(w[n][None, :] / grid[:, None]), -qmax, qmax)
                best = np.mean((wd - grid[:, None].astype(np.float64) * q) ** 2, axis=1).min()
                m_mm = _mse_np(w[n], s0, qmax)
                assert r["mse"][n] >= best * (1 - 1e-6)   # grid spacing 1.25e-5 relative
                assert r["mse"][n] <= m_mm
                gs.append(r["mse"][n] / best)
                gm.append(m_mm / best)
        assert np.median(gs) < np.median(gm) - 0.05
        assert max(gs) < 2.0


def test_ssz_rows_are_independent(orc):
    w = (np.random.default_rng(15).standard_normal((20, 64)) * 0.02).astype(np.float32)
    perm = np.random.default_rng(16).permutation(20)
    a = orc.ssz_quant_weight(w)
    b = orc.ssz_quant_weight(w[perm])
    np.testing.assert_array_equal(a["scale"][perm], b["scale"])
    np.testing.assert_array_equal(a["q"][perm], b["q"])


def test_ssz_fused_fold_equals_prefolded(orc):
    w = (np.random.default_rng(17).standard_normal((8, 32)) * 0.02).astype(np.float32)
    s = (np.random.default_rng(18).random(32) * 3 + 0.2).astype(np.float32)
    a = orc.ssz_quant_weight(w, s=s)
    b = orc.ssz_quant_weight(w * s[None, :])
    np.testing.assert_array_equal(a["scale"], b["scale"])


@pytest.mark.parametrize("bits", [8, 4])
def test_ssz_minimum_scale_floors_every_scale(orc, bits):
    # minimum scale 1e-5 (the page's algorithm parameters): weights of
    # magnitude ~1e-5 have least-squares optima below the floor, and every
    # returned scale must still be >= 1e-5, with the codes that scale implies.
    r = np.random.default_rng(27)
    w = (r.standard_normal((32, 64)) * 2e-5).astype(np.float32)
    out = orc.ssz_quant_weight(w, bits=bits)
    assert np.all(out["scale"] >= np.float32(1e-5))
    assert np.any(out["scale"] == np.float32(1e-5))
    qmax = (1 << (bits - 1)) - 1
    for n in range(32):
        np.testing.assert_array_equal(out["q"][n], _q(w[n], out["scale"][n], qmax).astype(np.int8))


def test_ssz_rejects_unsupported(orc):
    with pytest.raises(ValueError):
        orc.ssz_quant_weight(np.ones((2, 16), np.float32), bits=6)


# ----------------------------------------------------------------- step 4
def test_act_quant_golden_ties(orc):
    rows = [l.split() for l in open(os.path.join(GOLDEN, "act_round_half_even.txt"))
            if l.strip() and not l.startswith("#")]
    x = np.array([[float(a) for a, _ in rows]], np.float32)
    want = np.array([[int(b) for _, b in rows]], np.int8)
    q, sx = orc.quant_act_per_token(x)
    assert sx[0] == 1.0
    np.testing.assert_array_equal(q, want)


def test_act_quant_matches_numpy_rint(orc):
    x = _llm_like(40, 96, seed=19)
    inv = (np.random.default_rng(20).random(96) + 0.5).astype(np.float32)
    q, sx = orc.quant_act_per_token(x, inv)
    xs = x * inv[None, :]
    np.testing.assert_array_equal(sx, np.abs(xs).max(1) / np.float32(127))
    want = np.clip(np.rint(xs / sx[:, None]), -127, 127).astype(np.int8)
    np.testing.assert_array_equal(q, want)


def test_act_quant_error_bound_and_extremes(orc):
    x = _llm_like(64, 128, seed=21)
    q, sx = orc.quant_act_per_token(x)
    err = np.abs(x.astype(np.float64) - q.astype(np.float64) * sx[:, None].astype(np.float64))
    assert np.all(err <= sx[:, None] * (0.5 + 1e-6))
    # the row's absmax element lands on +/-127
    j = np.abs(x).argmax(1)
    assert np.all(np.abs(q[np.arange(64), j]) == 127)
    # sign is preserved
    assert np.all(np.sign(q) * np.sign(x) >= 0)


def test_act_quant_zero_row_and_identity_smoothing(orc):
    x = _llm_like(4, 32, seed=22)
    x[2] = 0.0
    q, sx = orc.quant_act_per_token(x)
    assert sx[2] == 0.0 and not q[2].any()
    q1, sx1 = orc.quant_act_per_token(x, np.ones(32, np.float32))
    np.testing.assert_array_equal(q, q1)
    np.testing.assert_array_equal(sx, sx1)


# ------------------------------------------------- asymmetric int8 SSZ
# "SSZ：权重量化算法说明": 初始化阶段 (MinMax min/max), 迭代优化阶段 (asymmetric:
# scale and offset by least squares), 收敛判断, 算法参数.
def _asym_codes_np(w, S, m):
    return np.clip(np.rint((w - np.float32(m)) / np.float32(S)), 0, 255)


def test_ssz_asym_minmax_init(orc):
    r = np.random.default_rng(40)
    w = (r.standard_normal((6, 96)) * 0.3 + 0.2).astype(np.float32)
    out = orc.ssz_quant_weight_asym(w, max_iters=0)
    np.testing.assert_array_equal(out["offset"], w.min(1))
    np.testing.assert_array_equal(out["scale"], (w.max(1) - w.min(1)) / np.float32(255))
    u = out["q"].astype(np.int32) + 128
    assert np.all(u[np.arange(6), w.argmin(1)] == 0) and np.all(u[np.arange(6), w.argmax(1)] == 255)
    for n in range(6):
        np.testing.assert_array_equal(u[n], _asym_codes_np(w[n], out["scale"][n], out["offset"][n]))


def test_ssz_asym_one_round_is_least_squares(orc):
    # one round by hand: codes at the MinMax pair, lstsq of w on [u, 1],
    # re-quantise, keep if better (numpy throughout)
    r = np.random.default_rng(41)
    w = (r.standard_normal((8, 200)) + 3.0).astype(np.float32)
    out = orc.ssz_quant_weight_asym(w, max_iters=1)
    for n in range(8):
        S0 = max((w[n].max() - w[n].min()) / np.float32(255), np.float32(1e-5))
        m0 = w[n].min()
        u = _asym_codes_np(w[n], S0, m0).astype(np.float64)
        a, b = np.linalg.lstsq(np.stack([u, np.ones_like(u)], 1), w[n].astype(np.float64), rcond=None)[0]
        Sc, mc = max(np.float32(a), np.float32(1e-5)), np.float32(b)

        def err(S, m):
            uu = _asym_codes_np(w[n], S, m).astype(np.float64)
            return np.mean((w[n].astype(np.float64) - (np.float64(S) * uu + np.float64(m))) ** 2)
        S_want, m_want = (Sc, mc) if err(Sc, mc) < err(S0, m0) else (S0, m0)
        np.testing.assert_allclose(out["scale"][n], S_want, rtol=1e-6)
        np.testing.assert_allclose(out["offset"][n], m_want, rtol=1e-6, atol=1e-6 * abs(m_want))


def test_ssz_asym_error_trace_and_codes(orc):
    r = np.random.default_rng(42)
    w = (r.standard_normal((12, 160)) * np.linspace(0.1, 2.0, 12)[:, None] + 0.5).astype(np.float32)
    out = orc.ssz_quant_weight_asym(w, trace=True)
    mm = orc.ssz_quant_weight_asym(w, max_iters=0)
    for n in range(12):
        u = _asym_codes_np(w[n], out["scale"][n], out["offset"][n])
        np.testing.assert_array_equal(out["q"][n].astype(np.int32) + 128, u)
        e = np.mean((w[n].astype(np.float64) - (np.float64(out["scale"][n]) * u + np.float64(out["offset"][n]))) ** 2)
        assert abs(out["mse"][n] - e) <= 1e-12 * e + 1e-30
        assert out["mse"][n] <= mm["mse"][n]
        assert np.all(np.diff(out["trace"][n]) <= 0)
    assert np.mean(out["mse"] < mm["mse"]) > 0.5


def test_ssz_asym_beats_symmetric_on_offset_rows(orc):
    r = np.random.default_rng(43)
    w = (r.standard_normal((16, 256)) + 10.0).astype(np.float32)  # far from zero
    a = orc.ssz_quant_weight_asym(w)
    sym = orc.ssz_quant_weight(w, bits=8)
    assert np.all(a["mse"] < 0.2 * sym["mse"])


def test_ssz_asym_scale_equivariance(orc):
    # w -> 2 w scales every fp operation exactly: codes equal, (S, m) double
    r = np.random.default_rng(44)
    w = (r.standard_normal((6, 128)) + 1.0).astype(np.float32)
    a = orc.ssz_quant_weight_asym(w, max_iters=3)
    b = orc.ssz_quant_weight_asym(2 * w, max_iters=3)
    np.testing.assert_array_equal(a["q"], b["q"])
    np.testing.assert_array_equal(2 * a["scale"], b["scale"])
    np.testing.assert_array_equal(2 * a["offset"], b["offset"])


def test_asym_codes_at_given_scale(orc):
    # hand-derived: S = 0.5, m = -1 (both exact); u = rint((w - m) / S)
    # clamped to [0, 255] with ties to even, stored as q = u - 128
    w = np.array([[0.25, 0.75, -1.0, -3.0, 126.75, 200.0, -0.75, 0.0]], np.float32)
    #       (w-m)/S:   2.5   3.5    0    -4   255.5   402    0.5   2
    want = np.array([[2, 4, 0, 0, 255, 255, 0, 2]], np.int32) - 128
    q = orc.weight_codes_asym(w, np.float32([0.5]), np.float32([-1.0]))
    np.testing.assert_array_equal(q, want)
    # the codes the searched (S, m) imply are the codes the search returns
    r = np.random.default_rng(46)
    w = (r.standard_normal((10, 144)) * 0.5 + 0.3).astype(np.float32)
    out = orc.ssz_quant_weight_asym(w)
    np.testing.assert_array_equal(orc.weight_codes_asym(w, out["scale"], out["offset"]), out["q"])
    # in range, each code reconstructs its weight within half a step
    u = orc.weight_codes_asym(w, out["scale"], out["offset"]).astype(np.float64) + 128
    rec = out["scale"][:, None].astype(np.float64) * u + out["offset"][:, None]
    inside = (u > 0) & (u < 255)
    assert np.all(np.abs(rec - w)[inside] <= 0.5 * out["scale"][:, None].repeat(144, 1)[inside] * (1 + 1e-6))


def test_act_rowsum_and_asym_dequant(orc):
    r = np.random.default_rng(45)
    qx = r.integers(-127, 128, (9, 64)).astype(np.int8)
    qw = r.integers(-128, 128, (7, 64)).astype(np.int8)
    sx = (r.random(9) * 0.1).astype(np.float32)
    S = (r.random(7) * 0.01).astype(np.float32)
    m = (r.standard_normal(7) * 0.1).astype(np.float32)
    R = orc.act_rowsum(qx)
    np.testing.assert_array_equal(R, qx.astype(np.int64).sum(1))
    acc = orc.gemm_i8(qx, qw)
    y = orc.dequant_asym(acc, R, sx, S, m, out="f32")
    A = (acc + 128 * R[:, None]).astype(np.float32)
    want = sx[:, None] * (S[None, :] * A + m[None, :] * R[:, None].astype(np.float32))
    np.testing.assert_array_equal(y, want)
    # the same as sum_k sx qx (S u + m) in fp64, up to fp32 rounding
    u = qw.astype(np.float64) + 128
    ref = sx[:, None].astype(np.float64) * (qx.astype(np.float64) @ (S[:, None] * u + m[:, None]).T)
    np.testing.assert_allclose(y, ref, rtol=1e-5, atol=1e-6 * np.abs(ref).max())


# ------------------------------------------------- row-parallel (K-sharded) linear
def test_given_scale_codes_match_numpy_and_per_token(orc):
    x = _llm_like(24, 96, seed=70)
    inv = (np.random.default_rng(71).random(96) + 0.5).astype(np.float32)
    q, sx = orc.quant_act_per_token(x, inv)
    np.testing.assert_array_equal(orc.quant_act_given_scale(x, inv, sx), q)
    sx2 = (sx * np.float32(0.6)).astype(np.float32)
    sx2[3] = 0.0
    with np.errstate(divide="ignore", invalid="ignore"):
        want = np.clip(np.rint((x * inv[None, :]) / sx2[:, None]), -127, 127)
    want[3] = 0
    np.testing.assert_array_equal(orc.quant_act_given_scale(x, inv, sx2), want.astype(np.int8))


def test_k_sharded_linear_equals_unsharded(orc):
    # per-shard scales, MAX, codes at the global scale, int32 SUM, dequant:
    # bit for bit the unsharded per-token path
    x = _llm_like(16, 128, seed=72)
    inv = (np.random.default_rng(73).random(128) + 0.5).astype(np.float32)
    qw = np.random.default_rng(74).integers(-127, 128, (40, 128)).astype(np.int8)
    sw = (np.random.default_rng(75).random(40) * 0.01).astype(np.float32)
    q, sx = orc.quant_act_per_token(x, inv)
    y_full = orc.dequant(orc.gemm_i8(q, qw), sx, sw, out="f32")
    cuts = [0, 48, 80, 128]
    sx_g = np.max([orc.quant_act_per_token(x[:, a:b], inv[a:b])[1] for a, b in zip(cuts, cuts[1:])], axis=0)
    np.testing.assert_array_equal(sx_g, sx)
    acc = sum(orc.gemm_i8(orc.quant_act_given_scale(x[:, a:b], inv[a:b], sx_g), qw[:, a:b])
              for a, b in zip(cuts, cuts[1:]))
    np.testing.assert_array_equal(orc.dequant(acc, sx_g, sw, out="f32"), y_full)


# ------------------------------------------------- LayerNorm fused with step 4
# SmoothQuant page section 1 (the scaling moves into the op that produces X);
# CUDA INT8 notes 4.2 (fuse quantization with the neighbouring kernel).
def _pairwise_golden():
    def val(t):
        return 2.0 ** int(t[2:]) if t.startswith("2^") else (-(2.0 ** int(t[3:])) if t.startswith("-2^")
                                                               else float(t))
    cases = []
    for line in open(os.path.join(GOLDEN, "pairwise_sum.txt")):
        if line.startswith("#") or not line.strip():
            continue
        f = line.split()
        k = int(f[1])
        cases.append((f[0], val(f[2]), np.array([val(t) for t in f[3:3 + k]])))
    return cases


def test_pairwise_sum_golden(orc):
    # see tests/golden/pairwise_sum.txt for the derivations
    cases = _pairwise_golden()
    assert [c[0] for c in cases] == ["A", "B", "C", "D"]
    for name, want, x in cases:
        assert orc.pairwise_sum(x) == want, name


def test_pairwise_sum_error_bound(orc):
    # within the pairwise-summation bound |S - s| <= g(ceil(log2 n)) sum|x|,
    # g(k) = k u / (1 - k u), u = 2^-53 (Higham), against the exact fsum;
    # exact on small integers
    r = np.random.default_rng(80)
    u = 2.0 ** -53
    for n in (1, 2, 3, 7, 8, 100, 1000, 4096, 5000):
        x = r.standard_normal(n) * np.exp(r.standard_normal(n) * 6)
        k = max(1, int(np.ceil(np.log2(n))))
        bound = k * u / (1 - k * u) * np.abs(x).sum()
        assert abs(orc.pairwise_sum(x) - math.fsum(x)) <= bound
        xi = r.integers(-1000, 1000, n).astype(np.float64)
        assert orc.pairwise_sum(xi) == xi.sum()


def test_layernorm_statistics_are_pairwise(orc):
    # rows of the golden cases A and B: mean and variance from the
    # hand-derived pairwise sums, the rest by the stated fp32 formulas
    cases = {c[0]: c[2] for c in _pairwise_golden()}
    for name, mean, ss in (("A", 0.25, 2.0 ** 107), ("B", 0.5, 2.0 ** 107)):
        # A: d = [2^53, 0.75, 0.75, -2^53] after rounding, squares sum to 2^107
        # B: d = [2^53, 0.5, 0.5, -2^53, 0.5, 0.5], sum 2^107 + 0.5 -> 2^107
        h = cases[name].astype(np.float32)[None, :]
        K = h.shape[1]
        _, _, y = orc.layernorm_quant(h, None, None, 0.0)
        r32 = np.float32(1.0 / np.sqrt(ss / K))
        want = (h[0] - np.float32(mean)) * r32
        np.testing.assert_array_equal(y[0], want)
    # row D's squares are golden case D: mean 0, var = (2 + 2^-51) / 16 exactly
    b = np.float32(2.0 ** -27)
    h = np.array([[1] + [b] * 7 + [-1] + [-b] * 7], np.float32)
    _, _, _, st = orc.layernorm_quant(h, None, None, 1e-5, stats=True)
    assert st[0, 0] == 0.0 and st[0, 1] == (2.0 + 2.0 ** -51) / 16
    assert math.fsum(cases["D"]) / 16 != st[0, 1]  # the exact sum would differ: the order is pinned


def test_layernorm_matches_torch_fp64(orc):
    r = np.random.default_rng(60)
    for scale, eps in ((3.0, 1e-5), (0.01, 1e-5), (1.0, 0.0)):
        h = (r.standard_normal((9, 96)) * scale + 0.5 * scale).astype(np.float32)
        g = (r.random(96) + 0.5).astype(np.float32)
        b = (r.standard_normal(96) * 0.1).astype(np.float32)
        _, _, y = orc.layernorm_quant(h, g, b, eps)
        want = torch.nn.functional.layer_norm(torch.from_numpy(h).double(), (96,), torch.from_numpy(g).double(),
                                              torch.from_numpy(b).double(), eps).numpy()
        # fp32 elementwise arithmetic after fp64 statistics: a few ulp of the fp64 result
        np.testing.assert_allclose(y, want.astype(np.float32), rtol=1e-6, atol=1e-6 * np.abs(want).max())


def test_layernorm_quant_composes_with_per_token_quant(orc):
    r = np.random.default_rng(61)
    h = _llm_like(20, 128, seed=62)
    g = (r.random(128) + 0.5).astype(np.float32)
    b = (r.standard_normal(128) * 0.1).astype(np.float32)
    inv = (r.random(128) + 0.25).astype(np.float32)
    q, sx, y = orc.layernorm_quant(h, g, b, 1e-5, inv)
    q2, sx2 = orc.quant_act_per_token(y, inv)
    np.testing.assert_array_equal(q, q2)
    np.testing.assert_array_equal(sx, sx2)


def test_layernorm_fold_of_smoothing_is_equivalent(orc):
    # diag(1/s) folded into gamma and beta gives the same codes up to rounding
    r = np.random.default_rng(63)
    h = _llm_like(32, 256, seed=64)
    g = (r.random(256) + 0.5).astype(np.float32)
    b = (r.standard_normal(256) * 0.1).astype(np.float32)
    inv = (r.random(256) * 2 + 0.1).astype(np.float32)
    q, sx, _ = orc.layernorm_quant(h, g, b, 1e-5, inv)
    qf, sxf, _ = orc.layernorm_quant(h, g * inv, b * inv, 1e-5)
    np.testing.assert_allclose(sxf, sx, rtol=1e-6)
    assert np.mean(q == qf) > 0.999 and np.abs(q.astype(int) - qf).max() <= 1


def test_layernorm_quant_constant_row(orc):
    h = np.full((2, 64), 3.25, np.float32)
    q, sx, y = orc.layernorm_quant(h, None, None, 1e-5)
    assert not y.any() and not q.any() and not sx.any()


# ------------------------------------------------- packed int4
def test_pack_int4_layout_and_round_trip(orc):
    # golden nibble layout: element 2i low, 2i+1 high, two's complement
    q = np.array([[1, -1, 7, -8, 0, 3, -2, 5]], np.int8)
    np.testing.assert_array_equal(orc.pack_int4(q)[0], np.array([0xF1, 0x87, 0x30, 0x5E], np.uint8))
    r = np.random.default_rng(50)
    q = r.integers(-8, 8, (13, 96)).astype(np.int8)
    p = orc.pack_int4(q)
    np.testing.assert_array_equal(p, ((q[:, 0::2].astype(np.int32) & 15) | ((q[:, 1::2].astype(np.int32) & 15) << 4)))
    np.testing.assert_array_equal(orc.unpack_int4(p, 96), q)
    # every byte value unpacks to a pair in [-8, 7] and packs back to itself
    allb = np.arange(256, dtype=np.uint8)[None, :]
    u = orc.unpack_int4(allb, 512)
    assert u.min() == -8 and u.max() == 7
    np.testing.assert_array_equal(orc.pack_int4(u), allb)


def test_w4a8_product_equals_int8_product_of_the_codes(orc):
    # the W4A8 GEMM is the int8 GEMM of the unpacked codes
    r = np.random.default_rng(51)
    qx = r.integers(-127, 128, (5, 64)).astype(np.int8)
    q4 = r.integers(-7, 8, (9, 64)).astype(np.int8)
    acc = orc.gemm_i8(qx, orc.unpack_int4(orc.pack_int4(q4), 64))
    np.testing.assert_array_equal(acc, qx.astype(np.int64) @ q4.astype(np.int64).T)


# ------------------------------------------------- static activation scale
# "PaddleNLP GPT 量化感知训练（QAT）实战指南" section 六 (moving_average_abs_max)
# and the CUDA INT8 notes section 2.1 (range calibration, saturation).
def test_static_batch_absmax_matches_numpy_and_column_route(orc):
    x = _llm_like(50, 96, seed=31)
    inv = (np.random.default_rng(32).random(96) + 0.25).astype(np.float32)
    a = orc.static_batch_absmax(x, inv)
    assert a == np.abs(x * inv[None, :]).max()
    # the same value from the per-channel absmax: |x| * c is monotonic in |x|
    assert a == (orc.calib_absmax(x) * inv).max()
    assert orc.static_batch_absmax(x) == np.abs(x).max()


def test_static_ema_closed_forms(orc):
    a = np.float32([3.0, 5.0, 2.0, 7.0])
    # rate 0: the last batch; rate 1: the first batch; first call sets the state
    assert orc.static_ema(123.0, 4.0, 0.9, first=True) == np.float32(4.0)
    m = a[0]
    for v in a[1:]:
        m = orc.static_ema(m, v, 0.0)
    assert m == a[-1]
    m = a[0]
    for v in a[1:]:
        m = orc.static_ema(m, v, 1.0)
    assert m == a[0]
    # rate 1/2 on small integers is exact: m = (((3+5)/2 + 2)/2 + 7)/2
    m = a[0]
    for v in a[1:]:
        m = orc.static_ema(m, v, 0.5)
    assert m == np.float32(((3.0 + 5.0) / 2 + 2.0) / 2 / 2 + 7.0 / 2)
    # general rate against the fp64 closed form rate^(T-1) a_1 + sum (1-rate) rate^(T-t) a_t
    r = np.random.default_rng(33)
    seq = (r.random(12) * 10).astype(np.float32)
    m = orc.static_range([np.full((1, 16), v, np.float32) for v in seq], rate=0.9)
    T = len(seq)
    want = 0.9 ** (T - 1) * float(seq[0]) + sum(0.1 * 0.9 ** (T - 1 - t) * float(seq[t]) for t in range(1, T))
    assert abs(float(m) - want) <= 1e-5 * want


def test_static_quant_matches_numpy_and_saturates(orc):
    x = _llm_like(24, 64, seed=34)
    inv = (np.random.default_rng(35).random(64) + 0.5).astype(np.float32)
    m = np.float32(np.abs(x * inv[None, :]).max() * np.float32(0.25))  # a range well below the max
    q = orc.quant_act_static(x, inv, m)
    S = orc.static_scale(m)
    assert S == m / np.float32(127)
    want = np.clip(np.rint((x * inv[None, :]) / S), -127, 127).astype(np.int8)
    np.testing.assert_array_equal(q, want)
    big = np.abs(x * inv[None, :]) > 128 * S
    assert big.any() and np.all(np.abs(q[big]) == 127)
    assert not orc.quant_act_static(x, inv, np.float32(0.0)).any()


def test_static_quant_equals_dynamic_at_the_row_range(orc):
    # with the static range equal to one row's abs-max, that row's codes are
    # the per-token codes (an independently pinned function)
    x = _llm_like(16, 80, seed=36)
    inv = (np.random.default_rng(37).random(80) + 0.5).astype(np.float32)
    qd, sx = orc.quant_act_per_token(x, inv)
    for t in (0, 7, 15):
        m = np.float32(sx[t] * np.float32(127))
        if orc.static_scale(m) != sx[t]:
            continue  # m / 127 does not round back to sx (rare); nothing to compare
        qs = orc.quant_act_static(x[t:t + 1], inv, m)
        np.testing.assert_array_equal(qs[0], qd[t])


# ----------------------------------------------------------------- step 5
@pytest.mark.parametrize("shape", [(1, 1, 16), (7, 5, 32), (33, 17, 48), (64, 64, 64)])
def test_gemm_matches_numpy_int64(orc, shape):
    M, N, K = shape
    r = np.random.default_rng(M * 1000 + N)
    qx = r.integers(-127, 128, size=(M, K), dtype=np.int8)
    qw = r.integers(-127, 128, size=(N, K), dtype=np.int8)
    want = qx.astype(np.int64) @ qw.astype(np.int64).T
    np.testing.assert_array_equal(orc.gemm_i8(qx, qw), want.astype(np.int32))


def test_gemm_operand_orientation(orc):
    # acc[t, n] uses row t of qx and row n of qw (both K-contiguous)
    qx = np.zeros((3, 16), np.int8)
    qw = np.zeros((5, 16), np.int8)
    qx[1, 4] = 3
    qw[2, 4] = -7
    acc = orc.gemm_i8(qx, qw)
    assert acc[1, 2] == -21 and np.count_nonzero(acc) == 1


def test_gemm_extremes_do_not_overflow(orc):
    K = 8192
    qx = np.full((2, K), 127, np.int8)
    qw = np.full((3, K), -127, np.int8)
    qw[1] = 127
    acc = orc.gemm_i8(qx, qw)
    assert acc[0, 0] == -K * 127 * 127 and acc[1, 1] == K * 127 * 127


def test_dequant_matches_library_casts(orc):
    r = np.random.default_rng(23)
    acc = r.integers(-2 ** 27, 2 ** 27, size=(9, 13), dtype=np.int32)
    sx = (r.random(9) * 0.1).astype(np.float32)
    sw = (r.random(13) * 1e-3).astype(np.float32)
    yf = orc.dequant(acc, sx, sw, out="f32")
    want = (acc.astype(np.float32) * sx[:, None]) * sw[None, :]
    np.testing.assert_array_equal(yf, want)
    yb = orc.dequant(acc, sx, sw, out="bf16")
    tb = torch.from_numpy(want).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(yb, tb)


def test_bf16_rounding_matches_torch(orc):
    r = np.random.default_rng(24)
    a = (r.standard_normal(4096) * 10.0 ** r.integers(-30, 30, 4096)).astype(np.float32)
    a[:4] = [0.0, -0.0, np.inf, -np.inf]
    # exact ties (low 16 bits 0x8000) with even and odd kept parts: RNE goes
    # to the even neighbour, which a round-half-up slip gets wrong
    ties = np.array([0x3F808000, 0x3F818000, 0xBF808000, 0xC0418000, 0x00018000, 0x7F7F8000],
                    dtype=np.uint32).view(np.float32)
    a[4:4 + ties.size] = ties
    want = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(orc.to_bf16_bits(a), want)


# ----------------------------------------------------------------- whole path
def test_smoothing_lowers_w8a8_error_with_outliers(orc):
    # the point of the method: with activation outlier channels, smoothing
    # (alpha = 0.5) gives a more accurate W8A8 product than no smoothing.
    x = _llm_like(64, 256, n_out=4, scale=50.0, seed=25)
    w = (np.random.default_rng(26).standard_normal((128, 256)) * 0.02).astype(np.float32)
    ref = x.astype(np.float64) @ w.astype(np.float64).T
    y_s = orc.linear(x, w, alpha=0.5, out="f32")["y"]
    y_0 = orc.linear(x, w, alpha=0.0, out="f32")["y"]      # alpha=0 still rescales; use s=1 below
    qw = orc.ssz_quant_weight(w)
    qx, sx = orc.quant_act_per_token(x)
    y_none = orc.dequant(orc.gemm_i8(qx, qw["q"]), sx, qw["scale"], out="f32")
    e = lambda y: np.linalg.norm(y - ref) / np.linalg.norm(ref)
    assert e(y_s) < 0.5 * e(y_none)
    assert e(y_s) < 0.05
    assert np.isfinite(y_0).all()
