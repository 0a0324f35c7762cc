"""The pins reject a wrong oracle.  Each case plants one plausible mistake
(a dropped term, a wrong sign, index, bit position or rounding rule) in a
copy of the C oracle, builds the copy, and runs the pin suite against it in
a subprocess: at least one pin must fail.  A control run of the unmodified
copy through the same route must pass.  CPU only."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE_C = os.path.join(ROOT, "oracle", "bitnet_oracle.c")
PINS = os.path.join(ROOT, "tests", "test_oracle_pins.py")

# (name, text in the oracle, replacement): each text occurs exactly once
MUTANTS = [
    # absmean gamma
    ("gamma_count_off_by_one", "double mean = s / (double)n;", "double mean = s / (double)(n + 1);"),
    ("gamma_exponent_off_by_one", "kulisch_add(acc, m | 0x800000u, (int)e - 1);",
     "kulisch_add(acc, m | 0x800000u, (int)e);"),
    ("gamma_sign_bit_kept", "bits &= 0x7fffffffu;                       /* |w| */", ""),
    # ternarise
    ("ternarise_eps_dropped", "float d = gamma + eps;", "float d = gamma;"),
    ("ternarise_round_half_away", "float r = rintf(t);", "float r = roundf(t);"),
    ("ternarise_truncate", "float r = rintf(t);", "float r = truncf(t);"),
    ("ternarise_clamp_sign", "else if (r <= -1.0f) q = -1;", "else if (r <= -1.0f) q = 1;"),
    # 2-bit pack / unpack
    ("pack_bit_order_reversed", "byte |= c << (2 * s);", "byte |= c << (2 * (3 - s));"),
    ("pack_index_transposed", "int64_t k = 16 * g + 4 * s + j;", "int64_t k = 16 * g + 4 * j + s;"),
    ("pack_code_negated", "if (q >= -1 && q <= 1) c = (unsigned)(q + 1);",
     "if (q >= -1 && q <= 1) c = (unsigned)(1 - q);"),
    ("unpack_code_negated", "else Wq[n * K + k] = (int8_t)((int)c - 1);",
     "else Wq[n * K + k] = (int8_t)(1 - (int)c);"),
    # activation quantiser
    ("act_scale_128", "float inv = 127.0f / a;", "float inv = 128.0f / a;"),
    ("act_floor_dropped", "if (a < floor_eps) a = floor_eps;", ""),
    ("act_truncate", "float v = rintf(t * inv);", "float v = truncf(t * inv);"),
    ("act_sum_of_magnitudes", "s += q;", "s += (q > 0 ? q : -q);"),
    ("rms_eps_dropped", "double r = 1.0 / sqrt(ss / (double)K + (double)rms_eps);",
     "double r = 1.0 / sqrt(ss / (double)K);"),
    ("rms_mean_over_k_minus_1", "double r = 1.0 / sqrt(ss / (double)K + (double)rms_eps);",
     "double r = 1.0 / sqrt(ss / (double)(K - 1) + (double)rms_eps);"),
    ("rms_scale_missing_absmax", "scale[m] = (float)(r * (double)a / 127.0);", "scale[m] = (float)(r / 127.0);"),
    # contraction and output
    ("linear_last_k_dropped", "for (int64_t k = 0; k < K; ++k)\n                s += (int64_t)xq",
     "for (int64_t k = 0; k + 1 < K; ++k)\n                s += (int64_t)xq"),
    ("output_scale_divided",
     "float sm = gamma * scale[m];\n        for (int64_t n = 0; n < N; ++n)\n            y[m * N + n] = (float)acc",
     "float sm = gamma / scale[m];\n        for (int64_t n = 0; n < N; ++n)\n            y[m * N + n] = (float)acc"),
    ("resid_subtracted", "y[m * N + n] = resid[m * N + n] + prod;", "y[m * N + n] = resid[m * N + n] - prod;"),
    # ReLU^2 gate
    ("relu_missing", "float r = (g > 0.0f) ? g : 0.0f;", "float r = g;"),
    ("gate_up_dropped", "t[i] = rr * up[i];", "t[i] = rr;"),
    # BitNet b1
    ("binarise_zero_to_minus", "Wb[i] = (W[i] >= 0.0f) ? (int8_t)1 : (int8_t)-1;",
     "Wb[i] = (W[i] > 0.0f) ? (int8_t)1 : (int8_t)-1;"),
    ("pack_b1_bit_order", "if (v == 1) word |= 1u << (8 * j + s);", "if (v == 1) word |= 1u << (8 * j + 7 - s);"),
    # base-3
    ("pack_t3_digit_layout", "int64_t k = 20 * g + 4 * i + j;\n                    int c = 1;",
     "int64_t k = 20 * g + 5 * j + i;\n                    int c = 1;"),
    # bf16 output rounding
    ("bf16_round_half_up", "u += 0x7fffu + lsb;", "u += 0x8000u;"),
]


def _run_pins(tmp_path, source: str) -> subprocess.CompletedProcess:
    src = tmp_path / "oracle_copy.c"
    src.write_text(source)
    env = dict(os.environ)
    env["BITNET_ORACLE_SRC"] = str(src)
    env["BITNET_ORACLE_LIB"] = str(tmp_path / "liboracle_copy.so")
    return subprocess.run([sys.executable, "-m", "pytest", PINS, "-x", "-q", "-p", "no:cacheprovider",
                           "-m", "not gpu"], env=env, cwd=ROOT, capture_output=True, text=True, timeout=900)


@pytest.fixture(scope="module")
def pin_runs(tmp_path_factory):
    """All pin runs (the control copy and every mutant), in parallel."""
    from concurrent.futures import ThreadPoolExecutor
    with open(ORACLE_C) as f:
        src = f.read()
    jobs = {"control": src}
    for name, old, new in MUTANTS:
        if src.count(old) == 1:
            jobs[name] = src.replace(old, new)
    with ThreadPoolExecutor(max_workers=max(1, min(8, os.cpu_count() or 1))) as ex:
        futs = {name: ex.submit(_run_pins, tmp_path_factory.mktemp(name), text) for name, text in jobs.items()}
        return {name: f.result() for name, f in futs.items()}


def test_control_copy_passes(pin_runs):
    r = pin_runs["control"]
    assert r.returncode == 0, r.stdout[-3000:]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_reject_planted_mistake(pin_runs, name, old, new):
    with open(ORACLE_C) as f:
        assert f.read().count(old) == 1, f"{name}: the text to change must occur exactly once"
    r = pin_runs[name]
    # pytest exit code 1: the run completed and at least one pin failed
    assert r.returncode == 1, f"{name}: no pin failed\n{r.stdout[-3000:]}"
