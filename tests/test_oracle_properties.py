"""Property-based pins for the CPU oracle (hypothesis, derandomised so every
run checks the same cases).  Each property is checked against something
other than the oracle: a round trip, a library routine (math.fsum, numpy's
int64 matmul), or an invariant of the method.  CPU only."""
import math

import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle

SETTINGS = settings(max_examples=60, deadline=None, derandomize=True,
                    suppress_health_check=[HealthCheck.too_slow, HealthCheck.data_too_large])

oracle.build()


@st.composite
def ternary(draw, k_step):
    N = draw(st.integers(1, 9))
    K = k_step * draw(st.integers(1, 12))
    seed = draw(st.integers(0, 2**31 - 1))
    return np.random.default_rng(seed).integers(-1, 2, (N, K)).astype(np.int8)


@SETTINGS
@given(ternary(16))
def test_pack_roundtrip(Wq):
    Wp, bad = oracle.pack(Wq)
    assert bad == 0 and Wp.shape == (Wq.shape[0], Wq.shape[1] // 4)
    assert np.array_equal(oracle.unpack(Wp, Wq.shape[1])[0], Wq)


@SETTINGS
@given(ternary(32))
def test_pack_b1_roundtrip(Wq):
    Wb = np.where(Wq >= 0, 1, -1).astype(np.int8)
    Wp, bad = oracle.pack_b1(Wb)
    assert bad == 0 and Wp.shape == (Wb.shape[0], Wb.shape[1] // 8)
    assert np.array_equal(oracle.unpack_b1(Wp, Wb.shape[1]), Wb)


@SETTINGS
@given(ternary(16))
def test_pack_t3_roundtrip(Wq):
    Wp, bad = oracle.pack_t3(Wq)
    assert bad == 0 and Wp.shape == (Wq.shape[0], oracle.t3_row_bytes(Wq.shape[1]))
    assert (Wp <= 242).all()
    assert np.array_equal(oracle.unpack_t3(Wp, Wq.shape[1])[0], Wq)


@SETTINGS
@given(st.integers(1, 6), st.integers(1, 20), st.integers(1, 9), st.integers(0, 2**31 - 1))
def test_contraction_is_the_integer_matmul(M, kb, N, seed):
    rng = np.random.default_rng(seed)
    K = 16 * kb
    xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
    Wq = rng.integers(-1, 2, (N, K)).astype(np.int8)
    ref = xq.astype(np.int64) @ Wq.astype(np.int64).T
    assert np.array_equal(oracle.linear_i32(xq, Wq).astype(np.int64), ref)


finite32 = st.floats(width=32, allow_nan=False, allow_infinity=False, min_value=-2.0 ** 100, max_value=2.0 ** 100)


@SETTINGS
@given(st.lists(finite32, min_size=1, max_size=200))
def test_gamma_is_correctly_rounded_mean(vals):
    W = np.array(vals, np.float32)
    ref = np.float32(math.fsum(abs(float(v)) for v in W) / W.size)
    assert np.float32(oracle.gamma(W)) == ref


@SETTINGS
@given(st.integers(1, 4), st.integers(1, 8), st.integers(0, 2**31 - 1), st.floats(1e-3, 1e3))
def test_quant_act_invariants(M, kb, seed, scale):
    rng = np.random.default_rng(seed)
    K = 16 * kb
    x = (rng.standard_normal((M, K)) * scale).astype(np.float32)
    x[rng.random((M, K)) < 0.2] = 0.0
    xq, s, xs = oracle.quant_act(x)
    assert xq.dtype == np.int8 and (np.abs(xq.astype(np.int32)) <= 127).all()
    assert np.array_equal(xs, xq.astype(np.int64).sum(1))
    for m in range(M):
        a = np.abs(x[m]).max()
        if a >= 1e-5:
            assert np.abs(xq[m].astype(np.int32)).max() == 127          # the row maximum maps to 127
            assert abs(float(s[m]) * 127.0 - a) <= 1e-6 * a               # scale = max|x| / 127
            # every code reconstructs its input within half a step
            err = np.abs(xq[m].astype(np.float64) * (a / 127.0) - x[m].astype(np.float64))
            assert (err <= 0.5 * a / 127.0 * (1 + 1e-5) + 1e-30).all()
        # codes carry the sign of their inputs
        assert (np.sign(xq[m]) * np.sign(x[m]) >= 0).all()


@SETTINGS
@given(st.integers(1, 6), st.integers(1, 8), st.integers(0, 2**31 - 1))
def test_ternarise_invariants(N, kb, seed):
    rng = np.random.default_rng(seed)
    K = 16 * kb
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    Wq, g = oracle.quant_weights(W)
    assert set(np.unique(Wq)).issubset({-1, 0, 1})
    assert (np.sign(Wq) * np.sign(W) >= 0).all()                 # no sign flips
    r = np.abs(W.astype(np.float64)) / (float(g) + 1e-8)
    assert (Wq[r < 0.499] == 0).all() and (Wq[r > 0.501] != 0).all()   # away from the 0.5 boundary
