"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of oracle/axon_ssm_oracle.c (a dropped
term, a wrong sign, a swapped operand, an index off by one, a reversed
order), builds it, and runs tests/test_oracle_pins.py against that build: at
least one pin must fail.  The real source is never modified.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "axon_ssm_oracle.c")

MUTANTS = {
    "dropped_D_skip": ("double y_ssm = acc + D[e] * u;", "double y_ssm = acc;"),
    "A_sign": ("A[n] = -exp(A_log[(size_t)e * N + n]);", "A[n] = exp(A_log[(size_t)e * N + n]);"),
    "C_replaced_by_B": ("acc += Cm[bn] * h[n];", "acc += Bm[bn] * h[n];"),
    "conv_taps_reversed": ("xc += conv_w[(size_t)e * K + k] * xpad[t + k];",
                           "xc += conv_w[(size_t)e * K + (K - 1 - k)] * xpad[t + k];"),
    "dt_lower_clip": ("#define ORACLE_DT_MIN 1e-4", "#define ORACLE_DT_MIN 1e-3"),
    "dt_upper_clip": ("#define ORACLE_DT_MAX 100.0", "#define ORACLE_DT_MAX 10.0"),
    "B_time_index_shift": ("size_t bn = ((size_t)b * L + t) * N + n;",
                           "size_t bn = ((size_t)b * L + (t > 0 ? t - 1 : 0)) * N + n;"),
    "gate_without_silu": ("y[idx] = y_ssm * oracle_silu(z[idx]);", "y[idx] = y_ssm * z[idx];"),
    "softplus_without_log1p": ("return log1p(exp(v));", "return exp(v);"),
    "cache_order_reversed": ("conv_cache_out[((size_t)b * KM1 + j) * E + e] = xpad[L + j];",
                             "conv_cache_out[((size_t)b * KM1 + j) * E + e] = xpad[L + KM1 - 1 - j];"),
    "input_before_decay": ("h[n] = abar * h[n] + bbar * u;", "h[n] = abar * (h[n] + bbar * u);"),
    "silu_as_sigmoid": ("double oracle_silu(double v) { return v / (1.0 + exp(-v)); }",
                        "double oracle_silu(double v) { return 1.0 / (1.0 + exp(-v)); }"),
    "conv_stage_taps_reversed": ("acc += conv_w[(size_t)e * K + k] * xv;",
                                 "acc += conv_w[(size_t)e * K + (K - 1 - k)] * xv;"),
    "conv_stage_cache_order": ("xv = conv_cache_in[((size_t)b * KM1 + (KM1 + s)) * E + e];",
                               "xv = conv_cache_in[((size_t)b * KM1 + (-1 - s)) * E + e];"),
    "ssd_input_without_dt": ("*s = a * *s + dt * xv[p] * Bt[n];", "*s = a * *s + xv[p] * Bt[n];"),
    "ssd_decay_sign": ("const double A = -exp(A_log[h]);", "const double A = exp(A_log[h]);"),
    "ssd_C_replaced_by_B": ("acc += *s * Ct[n];", "acc += *s * Bt[n];"),
    "ssd_dropped_D": ("yv[p] = acc + D[h] * xv[p];", "yv[p] = acc;"),
    "ssd_h0_ignored": ("S[i] = h0 ? h0[((size_t)b * H + h) * P * N + i] : 0.0;", "S[i] = 0.0;"),
    "ssd_input_before_decay": ("*s = a * *s + dt * xv[p] * Bt[n];", "*s = a * (*s + dt * xv[p] * Bt[n]);"),
    "ssd_output_before_update": ("*s = a * *s + dt * xv[p] * Bt[n];\n                        acc += *s * Ct[n];",
                                 "acc += *s * Ct[n];\n                        *s = a * *s + dt * xv[p] * Bt[n];"),
    "zoh_missing_A_division": ("double bbar = zoh ? expm1(dt * A[n]) / A[n] * Bm[bn] : dt * Bm[bn];",
                               "double bbar = zoh ? expm1(dt * A[n]) * Bm[bn] : dt * Bm[bn];"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor for {name} not found in the oracle source"
    mutated = tmp_path / "oracle_mutant.c"
    mutated.write_text(src.replace(old, new))
    lib = tmp_path / "liboracle_mutant.so"
    subprocess.run(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fno-fast-math",
                    "-ffp-contract=off", "-o", str(lib), str(mutated), "-lm"], check=True)
    env = dict(os.environ, AXON_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"no pin failed for the planted mistake {name}:\n{r.stdout[-2000:]}"
    assert "failed" in r.stdout


def test_unmutated_oracle_passes_the_pins(tmp_path):
    lib = tmp_path / "liboracle_copy.so"
    subprocess.run(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fno-fast-math",
                    "-ffp-contract=off", "-o", str(lib), SRC, "-lm"], check=True)
    env = dict(os.environ, AXON_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:]


def test_openmp_build_passes_the_pins(tmp_path):
    """The OpenMP build of the same source (channels spread over host cores)
    passes every pin, like the default single-threaded build."""
    lib = tmp_path / "liboracle_omp.so"
    subprocess.run(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fno-fast-math",
                    "-ffp-contract=off", "-fopenmp", "-o", str(lib), SRC, "-lm"], check=True)
    env = dict(os.environ, AXON_ORACLE_LIB=str(lib), OMP_NUM_THREADS="4")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:]
