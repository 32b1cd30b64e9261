"""Planted mistakes in the oracle must fail the pins.

Each case compiles a copy of ``oracle/w8a8_oracle.c`` with one plausible
mistake (a dropped term, a wrong sign, index or constant, a transposed
operand, another rounding rule) into a temporary directory and runs the pin
tests against it in a separate process; that run must fail (a crash counts
as a failure). Nothing here touches a GPU.
"""
import os
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "w8a8_oracle.c")

MUTATIONS = {
    "scale_denominator": ("S = a / 127.0f;", "S = a / 128.0f;"),
    "reciprocal_constant": ("r = 127.0f / a;", "r = 128.0f / a;"),
    "round_half_up": ("float t = nearbyintf(p);", "float t = floorf(p + 0.5f);"),
    "round_toward_zero": ("float t = nearbyintf(p);", "float t = truncf(p);"),
    "zero_point_sign_in_calibration": ("*Z = clamp_int(-128 - rne_clamped(lo * *r), -128, 127);",
                                       "*Z = clamp_int(-128 + rne_clamped(lo * *r), -128, 127);"),
    "range_without_lo": ("float d = hi - lo;", "float d = hi;"),
    "levels_254": ("*S = d / 255.0f;\n    *r = 255.0f / d;", "*S = d / 254.0f;\n    *r = 254.0f / d;"),
    "zero_point_subtracted_in_quant": ("rne_clamped(p) + Z, -128, 127", "rne_clamped(p) - Z, -128, 127"),
    "no_saturation_clamp": ("(int8_t)clamp_int(rne_clamped(p) + Z, -128, 127)", "(int8_t)(rne_clamped(p) + Z)"),
    "zero_point_correction_sign": ("if (z != 0) c -= z * (int64_t)colsum[n];",
                                   "if (z != 0) c += z * (int64_t)colsum[n];"),
    "per_row_scale_dropped": ("const float sx = s_x_per_row ? S_x[m] : S_x[0];", "const float sx = S_x[0];"),
    "weight_operand_transposed": ("s += (int64_t)Xq[m * K + k] * (int64_t)Wq[n * K + k];",
                                  "s += (int64_t)Xq[m * K + k] * (int64_t)Wq[k * N + n];"),
    "bias_dropped": ("if (bias) add = add + bias[n];", "if (bias) add = add;"),
    "epilogue_unfused": ("y[m * N + n] = fmaf(f, sc, add);", "y[m * N + n] = f * sc + add;"),
    "colsum_of_first_row": ("for (int64_t k = 0; k < K; ++k) s += Wq[n * K + k];",
                            "for (int64_t k = 0; k < K; ++k) s += Wq[k];"),
    "threshold_not_strict": ("X[m * ldx + k])) > threshold", "X[m * ldx + k])) >= threshold"),
    "side_weight_row_index": ("W[(int64_t)idx[j] * ldw + n]", "W[(int64_t)j * ldw + n]"),
    "outliers_kept_in_row_scale": ("if (skip && skip[i]) continue;", ""),
    "bf16_round_half_away": ("u += 0x7fffu + keep_lsb;", "u += 0x8000u;"),
    "dequant_zero_point_added": ("float y = S * (float)((int32_t)Xq[m * K + k] - Z);",
                                 "float y = S * (float)((int32_t)Xq[m * K + k] + Z);"),
    "tiny_vector_scale_overflow_unchecked": ("if (a > 0.0f && 127.0f / a <= FLT_MAX) {", "if (a > 0.0f) {"),
    "tiny_range_calibration_unchecked": ("if (hi == lo || !(255.0f / d <= FLT_MAX)) {", "if (hi == lo) {"),
    "weight_read_along_rows": ("absmax_quant_vector(W, dtype, n, ldw, K, NULL, Wq + n * K, 1, &s_w[n]);",
                               "absmax_quant_vector(W, dtype, n, 1, K, NULL, Wq + n * K, 1, &s_w[n]);"),
}


def _run_pins_against(name, tmpdir):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    if old not in src:
        return name, "anchor not found"
    c = os.path.join(tmpdir, f"{name}.c")
    so = os.path.join(tmpdir, f"lib{name}.so")
    with open(c, "w") as f:
        f.write(src.replace(old, new, 1))
    subprocess.run(["gcc", *oracle._CFLAGS, c, "-o", so, "-lm"], check=True)
    env = dict(os.environ, ORACLE_LIB_OVERRIDE=so, OMP_NUM_THREADS="1")
    proc = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                           os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return name, ("caught" if proc.returncode != 0 else "NOT caught")


def test_every_planted_mistake_fails_a_pin():
    with tempfile.TemporaryDirectory() as d:
        with ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as ex:
            results = dict(ex.map(lambda n: _run_pins_against(n, d), sorted(MUTATIONS)))
    missed = {k: v for k, v in results.items() if v != "caught"}
    assert not missed, missed
