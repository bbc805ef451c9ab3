"""Mutation check of the oracle's pins.

Each case plants one plausible slip in a copy of oracle/oracle.c (a dropped
term, a wrong sign or exponent, a transposed operand, a wrong rounding mode,
an off-by-one range), builds it on the CPU, and runs the pins of
tests/test_oracle_pins.py against it.  At least one pin must fail for every
planted slip; the unmodified source must pass them all.

Not planted: dropping the greedy keep-if-better test of the SSZ search.  In
exact arithmetic it never rejects: the least-squares candidate minimises the
residual for the current codes, and re-rounding at the candidate scale gives
each element its nearest code, so the candidate's error is never larger.  The
keep only matters at fp rounding ties, so that mutant is equivalent.
"""
import inspect
import os

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = open(os.path.join(os.path.dirname(oracle.__file__), "oracle.c")).read()

# (name, original text, replacement)
MUTANTS = [
    ("calib_drops_abs", "float a = fabsf(row[j]);", "float a = row[j];"),
    ("smooth_weight_exponent_is_alpha", "pow((double)aw[j], 1.0 - a)", "pow((double)aw[j], a)"),
    ("smooth_swaps_x_and_w", "pow((double)ax[j], a) / pow((double)aw[j], 1.0 - a)",
     "pow((double)aw[j], a) / pow((double)ax[j], 1.0 - a)"),
    ("fold_wrong_column", "out[r * K + j] = a[r * K + j] * f[j];",
     "out[r * K + j] = a[r * K + j] * f[(j + 1) % K];"),
    ("round_half_away", "float r = rintf(w / s);", "float r = roundf(w / s);"),
    ("asymmetric_clamp", "if (r < -(float)qmax)\n        r = -(float)qmax;",
     "if (r < -(float)(qmax + 1))\n        r = -(float)(qmax + 1);"),
    ("mse_is_sum_not_mean", "(double)sym_code(w[k], s, qmax);\n        acc += e * e;\n    }\n    return acc / (double)K;",
     "(double)sym_code(w[k], s, qmax);\n        acc += e * e;\n    }\n    return acc;"),
    ("asym_mse_is_sum_not_mean", "(double)m);\n        acc += e * e;\n    }\n    return acc / (double)K;",
     "(double)m);\n        acc += e * e;\n    }\n    return acc;"),
    ("ls_inverted", "s_cand = (float)(num / (double)den);", "s_cand = (float)((double)den / num);"),
    ("ls_drops_square", "den += (int64_t)q * (int64_t)q;", "den += (int64_t)(q < 0 ? -q : q);"),
    ("convergence_sign_flipped", "(delta / m_best < SSZ_CONVERGE_THRESHOLD)",
     "(delta / m_best > SSZ_CONVERGE_THRESHOLD)"),
    ("minmax_uses_qmax_plus_one", "float s_best = amax / (float)qmax;",
     "float s_best = amax / (float)(qmax + 1);"),
    ("candidate_not_floored",
     "s_cand = (float)(num / (double)den);\n            if (s_cand < SSZ_MIN_SCALE)\n                s_cand = SSZ_MIN_SCALE;",
     "s_cand = (float)(num / (double)den);"),
    ("act_scale_128", "float s = amax / (float)ACT_QMAX;\n        sx[t] = s;\n        for (int64_t j = 0; j < K; ++j) {\n            float v = inv_s",
     "float s = amax / 128.0f;\n        sx[t] = s;\n        for (int64_t j = 0; j < K; ++j) {\n            float v = inv_s"),
    ("ln_act_scale_128", "float s = amax / (float)ACT_QMAX;\n        sx[t] = s;\n        for (int64_t j = 0; j < K; ++j)\n            q[t * K + j] = (s == 0.0f) ? (int8_t)0 : (int8_t)sym_code(y[j]",
     "float s = amax / 128.0f;\n        sx[t] = s;\n        for (int64_t j = 0; j < K; ++j)\n            q[t * K + j] = (s == 0.0f) ? (int8_t)0 : (int8_t)sym_code(y[j]"),
    ("act_divides_by_inv_s", "float v = inv_s ? row[j] * inv_s[j] : row[j];\n            q[",
     "float v = inv_s ? row[j] / inv_s[j] : row[j];\n            q["),
    ("gemm_transposed_weight", "(int64_t)qw[n * K + k]", "(int64_t)qw[k * N + n]"),
    ("dequant_drops_token_scale", "((float)acc[t * N + n] * sx[t]) * sw[n]",
     "((float)acc[t * N + n]) * sw[n]"),
    ("bf16_rounds_half_up", "u += 0x7fffu + ((u >> 16) & 1u);", "u += 0x8000u;"),
    ("static_ema_swaps_weights", "float keep = rate * state;\n    float w = 1.0f - rate;",
     "float keep = (1.0f - rate) * state;\n    float w = rate;"),
    ("static_ema_ignores_first", "    if (first)\n        return a;\n", ""),
    ("static_range_drops_smoothing", "float v = inv_s ? x[t * K + j] * inv_s[j] : x[t * K + j];\n            float a",
     "float v = x[t * K + j];\n            float a"),
    ("static_scale_128", "float S = m / (float)ACT_QMAX;", "float S = m / 128.0f;"),
    ("asym_code_ignores_offset", "float v = w - m;", "float v = w;"),
    ("asym_ls_offset_sign", "double b = (sw - a * (double)su) / (double)K;",
     "double b = (sw + a * (double)su) / (double)K;"),
    ("asym_minmax_254_levels", "float s_best = (wmax - wmin) / (float)ASYM_UMAX;",
     "float s_best = (wmax - wmin) / 254.0f;"),
    ("asym_dequant_drops_128R", "int32_t A = acc[t * N + n] + 128 * R[t];", "int32_t A = acc[t * N + n];"),
    ("asym_dequant_drops_offset", "float y = sx[t] * (p + o);", "float y = sx[t] * p;"),
    ("given_scale_ignores_smoothing", "float v = inv_s ? x[t * K + j] * inv_s[j] : x[t * K + j];\n            q[t * K + j] = (sx[t] == 0.0f)",
     "float v = x[t * K + j];\n            q[t * K + j] = (sx[t] == 0.0f)"),
    ("ln_drops_eps", "double rstd = 1.0 / sqrt(ss / (double)K + (double)eps);",
     "double rstd = 1.0 / sqrt(ss / (double)K);"),
    ("ln_unbiased_variance", "double rstd = 1.0 / sqrt(ss / (double)K + (double)eps);",
     "double rstd = 1.0 / sqrt(ss / (double)(K - 1) + (double)eps);"),
    ("ln_drops_beta", "float b = beta ? beta[j] : 0.0f;", "float b = 0.0f;"),
    ("ln_smooths_before_norm", "float v = inv_s ? yj * inv_s[j] : yj;", "float v = yj;"),
    ("ln_sequential_mean", "double mu = oracle_pairwise_sum(tmp, K) / (double)K;",
     "double mu = 0.0;\n        for (int64_t j = 0; j < K; ++j)\n            mu += tmp[j];\n        mu /= (double)K;"),
    ("ln_sequential_variance", "double ss = oracle_pairwise_sum(tmp, K);",
     "double ss = 0.0;\n        for (int64_t j = 0; j < K; ++j)\n            ss += tmp[j];"),
    ("pairwise_unpadded_split", "while (P < K)\n        P *= 2;", "P = K;"),
    ("asym_given_codes_not_offset", "q[n * K + k] = (int8_t)((int)asym_code(w[n * K + k], S[n], m[n]) - 128);",
     "q[n * K + k] = (int8_t)((int)asym_code(w[n * K + k], S[n], m[n]) - 127);"),
    ("int4_nibbles_swapped", "packed[n * (K / 2) + i] = (uint8_t)(lo | (hi << 4));",
     "packed[n * (K / 2) + i] = (uint8_t)(hi | (lo << 4));"),
    ("int4_unpack_no_sign", "q[n * K + 2 * i] = (int8_t)(lo >= 8 ? lo - 16 : lo);", "q[n * K + 2 * i] = (int8_t)lo;"),
]

PIN_TESTS = []
for _name, _fn in inspect.getmembers(pins, inspect.isfunction):
    if not _name.startswith("test_"):
        continue
    marks = getattr(_fn, "pytestmark", [])
    params = [m for m in marks if m.name == "parametrize"]
    if params:
        argname, values = params[0].args
        for v in values:
            PIN_TESTS.append((f"{_name}[{v}]", _fn, {argname: v}))
    else:
        PIN_TESTS.append((_name, _fn, {}))


# the brute-force grid is the slowest pin: run it last
PIN_TESTS.sort(key=lambda t: "brute_force" in t[0])


def _failing_pins(stop_at_first: bool = False):
    failed = []
    for name, fn, kw in PIN_TESTS:
        try:
            fn(oracle, **kw)
        except Exception:  # an assertion, or a crash-free numeric error
            failed.append(name)
            if stop_at_first:
                break
    return failed


@pytest.fixture(scope="module")
def workdir(tmp_path_factory):
    return tmp_path_factory.mktemp("oracle_mutants")


def test_unmodified_oracle_passes_every_pin(workdir):
    path = oracle.build_variant(SRC, str(workdir / "lib_orig.so"))
    oracle.load_library(path)
    try:
        assert _failing_pins() == []
    finally:
        oracle.load_library(None)


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_slip_is_caught(workdir, name, old, new):
    assert SRC.count(old) == 1, "mutation site not unique: %s" % name
    path = oracle.build_variant(SRC.replace(old, new), str(workdir / ("lib_%s.so" % name)))
    oracle.load_library(path)
    try:
        failed = _failing_pins(stop_at_first=True)
    finally:
        oracle.load_library(None)
    assert failed, "no pin caught the planted slip %s" % name
