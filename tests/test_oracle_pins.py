"""Pins for the CPU oracle: each test checks the oracle against something other
than itself -- a hand-worked example from the pages' formulas, a closed form,
an invariant, a library routine or brute force.  CPU only."""
import math

import numpy as np
import pytest
import torch

from conftest import golden_lines

from bitlinear_bitnet_linear_b200 import synthetic


def _floats(s):
    return np.array([float(v) for v in s.split()], np.float64)


# --------------------------------------------------------------------------
# absmean scale gamma
# --------------------------------------------------------------------------

def _abs_arrays():
    rng = np.random.default_rng(7)
    yield rng.normal(0, 0.02, 100_003).astype(np.float32)
    # wide dynamic range including subnormals, huge values and exact zeros
    e = rng.integers(-149, 120, 50_000)
    v = (rng.random(50_000) + 0.5) * np.exp2(e.astype(np.float64))
    v = v.astype(np.float32) * np.where(rng.random(50_000) < 0.5, -1, 1).astype(np.float32)
    v[::97] = 0.0
    yield v
    # cancellation-prone: one big value and many tiny ones
    w = np.full(20_000, 1e-30, np.float32)
    w[0] = 3e30
    yield w
    yield np.array([np.float32(1.4e-45)] * 7, np.float32)       # subnormal min


def test_abs_sum_is_correctly_rounded(orc):
    """math.fsum is a correctly rounded sum; the oracle's exact accumulator must
    agree bit for bit (a dropped carry, limb or sticky bit fails here)."""
    for W in _abs_arrays():
        ref = math.fsum(np.abs(W.astype(np.float64)).tolist())
        assert orc.abs_sum(W) == ref


def test_gamma_is_rounded_mean(orc):
    for W in _abs_arrays():
        ref = np.float32(math.fsum(np.abs(W.astype(np.float64)).tolist()) / W.size)
        assert orc.gamma(W) == ref


def test_gamma_statistics():
    """For W ~ N(0, s), E|W| = s*sqrt(2/pi): 0.015958 at s = 0.02."""
    import oracle
    W = synthetic.latent_weights(2048, 2048, seed=3).numpy()
    g = float(oracle.gamma(W))
    mu = 0.02 * math.sqrt(2 / math.pi)
    sd = 0.02 * math.sqrt(1 - 2 / math.pi) / math.sqrt(W.size)
    assert abs(g - mu) < 6 * sd


def test_gamma_zero(orc):
    assert orc.gamma(np.zeros((4, 16), np.float32)) == 0.0


# --------------------------------------------------------------------------
# ternarisation
# --------------------------------------------------------------------------

def test_ternarise_golden(orc):
    for line in golden_lines("ternarise_examples.txt"):
        name, shape, w, g, q = [s.strip() for s in line.split("|")]
        N, K = map(int, shape.split())
        W = _floats(w).astype(np.float32).reshape(N, K)
        Wq, gam = orc.quant_weights(W)
        assert np.isclose(float(gam), float(g), rtol=1e-6), name
        assert (Wq.reshape(-1) == _floats(q).astype(np.int8)).all(), name


def test_ternarise_ties_to_even(orc):
    """With gamma = 1 exactly (d = 1 + 1e-8 rounds to 1), W/d = W, so the
    half-way values pin torch.round's ties-to-even."""
    W = np.array([0.5, -0.5, 1.5, -1.5, 0.49999997, 0.50000006, 2.5, -2.5], np.float32)
    q = orc.ternarise(W, np.float32(1.0))
    assert q.tolist() == [0, 0, 1, -1, 0, 1, 1, -1]


def test_ternarise_invariants(orc):
    W = synthetic.latent_weights(257, 320, seed=11).numpy()
    Wq, g = orc.quant_weights(W)
    assert set(np.unique(Wq).tolist()) <= {-1, 0, 1}
    Wq2 = orc.ternarise(-W, g)
    assert (Wq2 == -Wq).all()                       # odd symmetry


def test_ternarise_idempotent(orc):
    """W = c*T with ternary T of zero fraction z < 1: gamma = c(1-z), nonzeros
    map to 1/(1-z) >= 1 -> clamp 1, so quantising returns T exactly."""
    rng = np.random.default_rng(5)
    for z in (0.0, 0.3, 0.9):
        T = rng.choice([-1, 1], size=(64, 96)).astype(np.int8)
        T[rng.random(T.shape) < z] = 0
        c = np.float32(0.037)
        Wq, g = orc.quant_weights(T.astype(np.float32) * c)
        assert (Wq == T).all()
        nz = np.count_nonzero(T)
        assert np.isclose(float(g), float(c) * nz / T.size, rtol=1e-6)


def test_ternarise_constant(orc):
    for c, expect in ((0.25, 1), (-3.0, -1)):
        Wq, g = orc.quant_weights(np.full((3, 16), c, np.float32))
        assert g == np.float32(abs(c)) and (Wq == expect).all()


def test_ternarise_all_zero(orc):
    Wq, g = orc.quant_weights(np.zeros((5, 32), np.float32))
    assert g == 0 and (Wq == 0).all()


def test_zero_fraction_statistics(orc):
    """Zero fraction for Gaussian W: P(|W| < gamma/2) with gamma = s*sqrt(2/pi)
    is erf(0.5*sqrt(2/pi)/sqrt(2)) = 0.3101 (the '~1/3 zeros' of b1.58)."""
    W = synthetic.latent_weights(1024, 2048, seed=9).numpy()
    Wq, _ = orc.quant_weights(W)
    z = float((Wq == 0).mean())
    expect = math.erf(0.5 * math.sqrt(2 / math.pi) / math.sqrt(2))
    assert abs(z - expect) < 0.003


# --------------------------------------------------------------------------
# 2-bit pack
# --------------------------------------------------------------------------

def test_pack_golden(orc):
    for line in golden_lines("pack_layout.txt"):
        k, ent, hexs = [s.strip() for s in line.split("|")]
        K = int(k)
        q = np.zeros((1, K), np.int8)
        for e in ent.split():
            a, b = e.split(":")
            if a == "all":
                q[:] = int(b)
            else:
                q[0, int(a)] = int(b)
        packed, bad = orc.pack(q)
        assert bad == 0
        assert packed.reshape(-1).tolist() == [int(h, 16) for h in hexs.split()]


def test_pack_size_and_no_code3(orc):
    rng = np.random.default_rng(1)
    for N, K in ((1, 16), (3, 48), (17, 272), (64, 2560)):
        q = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
        p, bad = orc.pack(q)
        assert bad == 0 and p.shape == (N, K // 4) and p.nbytes == N * K // 4
        fields = np.stack([(p >> (2 * s)) & 3 for s in range(4)])
        assert not (fields == 3).any()


def test_pack_roundtrip_exhaustive(orc):
    """All 3^8 patterns in each half of a 16-weight group (the other half
    fixed to each constant), plus random rows: unpack(pack(q)) == q."""
    vals = np.array(np.meshgrid(*[[-1, 0, 1]] * 8, indexing="ij")).reshape(8, -1).T
    rows = []
    for fill in (-1, 0, 1):
        a = np.full((vals.shape[0], 16), fill, np.int8)
        a[:, :8] = vals
        b = np.full((vals.shape[0], 16), fill, np.int8)
        b[:, 8:] = vals
        rows += [a, b]
    q = np.concatenate(rows)
    p, bad = orc.pack(q)
    back, bad2 = orc.unpack(p, 16)
    assert bad == 0 and bad2 == 0 and (back == q).all()
    rng = np.random.default_rng(2)
    q = rng.integers(-1, 2, size=(33, 2560 + 16)).astype(np.int8)
    back, _ = orc.unpack(orc.pack(q)[0], q.shape[1])
    assert (back == q).all()


def test_pack_invalid_counted(orc):
    q = np.zeros((2, 16), np.int8)
    q[0, 3] = 2
    q[1, 7] = -5
    p, bad = orc.pack(q)
    assert bad == 2
    back, bad2 = orc.unpack(p, 16)
    assert bad2 == 2 and back[0, 3] == 0 and back[1, 7] == 0


# --------------------------------------------------------------------------
# activation quantisation
# --------------------------------------------------------------------------

def test_quant_act_golden(orc):
    lines = golden_lines("quant_act_examples.txt")
    x = np.stack([_floats(l.split("|")[0]) for l in lines]).astype(np.float32)
    xq, sc, xs = orc.quant_act(x)
    for i, l in enumerate(lines):
        _, q, s, frac = [t.strip() for t in l.split("|")]
        assert xq[i].tolist() == [int(v) for v in q.split()]
        assert xs[i] == int(s)
        a, b = frac.split("/")
        assert sc[i] == np.float32(np.float32(float(a)) / np.float32(float(b)))


def test_quant_act_invariants(orc):
    x = synthetic.activations(9, 2560, seed=4, dtype=torch.float32).numpy()
    xq, sc, xs = orc.quant_act(x)
    assert xq.min() >= -127 and xq.max() <= 127          # -128 is unreachable
    assert (np.abs(xq).max(axis=1) == 127).all()
    assert (xs == xq.astype(np.int64).sum(axis=1)).all()
    assert np.allclose(sc * 127, np.abs(x).max(axis=1), rtol=1e-6)
    # power-of-two rescaling commutes exactly with the quantiser
    xq2, sc2, _ = orc.quant_act(x * np.float32(8.0))
    assert (xq2 == xq).all() and (sc2 == sc * 8).all()


def test_quant_act_integer_identity(orc):
    rng = np.random.default_rng(3)
    x = rng.integers(-127, 128, size=(4, 64)).astype(np.float32)
    x[:, 5] = 127
    xq, sc, _ = orc.quant_act(x)
    assert (xq == x.astype(np.int8)).all() and (sc == 1).all()


def test_quant_act_norm(orc):
    """With unit gain the norm leaves the codes unchanged and multiplies the
    scale by r = 1/sqrt(mean x^2 + eps); a general gain equals quantising x*g."""
    x = synthetic.activations(5, 2560, seed=6, dtype=torch.float32).numpy()
    g = np.ones(2560, np.float32)
    xq0, sc0, xs0 = orc.quant_act(x)
    xq1, sc1, xs1 = orc.quant_act(x, g, 1e-5)
    assert (xq0 == xq1).all() and (xs0 == xs1).all()
    xd = x.astype(np.float64)
    r = 1.0 / np.sqrt((xd * xd).mean(axis=1) + np.float64(np.float32(1e-5)))
    assert np.allclose(sc1, r * sc0.astype(np.float64), rtol=2e-7)
    gain = np.random.default_rng(8).uniform(0.5, 1.5, 2560).astype(np.float32)
    xq2, _, _ = orc.quant_act(x, gain, 1e-5)
    xq3, _, _ = orc.quant_act(x * gain)
    assert (xq2 == xq3).all()


def test_quant_act_norm_constant_row(orc):
    """x = c * ones: r = 1/sqrt(c^2 + eps), all codes 127, scale = r*c/127."""
    c = 0.75
    x = np.full((1, 64), c, np.float32)
    xq, sc, xs = orc.quant_act(x, np.ones(64, np.float32), 1e-5)
    assert (xq == 127).all() and xs[0] == 127 * 64
    r = 1 / math.sqrt(c * c + float(np.float32(1e-5)))
    assert sc[0] == np.float32(r * c / 127)


# --------------------------------------------------------------------------
# contraction and output
# --------------------------------------------------------------------------

def _rand_q(M, N, K, seed):
    rng = np.random.default_rng(seed)
    xq = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    Wq = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    return xq, Wq


def test_linear_add_subtract_identity(orc):
    xq, Wq = _rand_q(7, 33, 448, 12)
    acc = orc.linear_i32(xq, Wq)
    x = xq.astype(np.int64)
    plus = np.stack([(x * (Wq[n] == 1)).sum(1) for n in range(Wq.shape[0])], 1)
    minus = np.stack([(x * (Wq[n] == -1)).sum(1) for n in range(Wq.shape[0])], 1)
    assert (acc == plus - minus).all()


def test_linear_code_offset_identity(orc):
    """acc = sum_k c*x - sum_k x with c = q + 1 (the stored 2-bit code)."""
    xq, Wq = _rand_q(3, 40, 512, 13)
    acc = orc.linear_i32(xq, Wq)
    c = (Wq.astype(np.int64) + 1)
    x = xq.astype(np.int64)
    assert (acc == x @ c.T - x.sum(1, keepdims=True)).all()


def test_linear_vs_float64_matmul(orc):
    xq, Wq = _rand_q(16, 64, 6912, 14)
    acc = orc.linear_i32(xq, Wq)
    ref = xq.astype(np.float64) @ Wq.astype(np.float64).T    # exact below 2^53
    assert (acc.astype(np.float64) == ref).all()


def test_linear_bruteforce_tiny(orc):
    xq, Wq = _rand_q(2, 3, 32, 15)
    acc = orc.linear_i32(xq, Wq)
    for m in range(2):
        for n in range(3):
            s = 0
            for k in range(32):
                s += int(xq[m, k]) * int(Wq[n, k])
            assert acc[m, n] == s


def test_linear_golden(orc):
    d = {}
    for line in golden_lines("linear_example.txt"):
        parts = [p.strip() for p in line.split("|")]
        d[parts[0]] = [_floats(p) for p in parts[1:]]
    xq = np.stack(d["xq"]).astype(np.int8)
    wq = np.stack(d["wq"]).astype(np.int8)
    acc = orc.linear_i32(xq, wq)
    assert (acc == np.stack(d["acc"]).astype(np.int32)).all()
    y = orc.output(acc, np.float32(d["gamma"][0][0]), d["scale"][0].astype(np.float32))
    assert (y == np.stack(d["y"]).astype(np.float32)).all()


def test_output_vs_dequantised_matmul(orc):
    """y against a float64 product of the dequantised operands
    (x_q * s) @ (W_q * gamma)^T."""
    x = synthetic.activations(6, 2560, seed=21, dtype=torch.float32).numpy()
    W = synthetic.latent_weights(300, 2560, seed=22).numpy()
    Wq, g = orc.quant_weights(W)
    y, xq, sc, _, _ = orc.bitlinear(x, Wq, g)
    ref = (xq.astype(np.float64) * sc[:, None]) @ (Wq.astype(np.float64) * float(g)).T
    assert np.allclose(y, ref, rtol=1e-6, atol=1e-12 * np.abs(ref).max())


def test_bf16_rounding_matches_torch(orc):
    rng = np.random.default_rng(30)
    v = rng.normal(0, 10, 200_000).astype(np.float32)
    # exact ties: bf16 value plus half an ulp
    base = torch.from_numpy(v[:1000]).to(torch.bfloat16).float().numpy()
    ties = (base.view(np.uint32) | np.uint32(0x8000)).view(np.float32)
    v = np.concatenate([v, ties, np.array([0.0, -0.0, 3.4e38, -3.4e38, 1e-40], np.float32)])
    ours = orc.to_bf16_bits(v)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert (ours == ref).all()


# ---------------------------------------------------------------------------
# ReLU^2 gate and residual output ("Key Technologies ...", Architectural
# Innovations: squared ReLU in the feed-forward layers).
# ---------------------------------------------------------------------------
def test_relu2_golden(orc):
    rows = [ln.split() for ln in golden_lines("relu2_examples.txt")]
    g = np.array([float(r[0]) for r in rows], np.float32)
    u = np.array([float(r[1]) for r in rows], np.float32)
    want = np.array([float(r[2]) for r in rows], np.float32)
    got = orc.relu2_gate(g, u)
    assert np.array_equal(got, want), (got, want)


def test_relu2_invariants(orc):
    rng = np.random.default_rng(7)
    g = rng.standard_normal(20000).astype(np.float32) * 3
    u = rng.standard_normal(20000).astype(np.float32) * 3
    t = orc.relu2_gate(g, u)
    assert np.all(t[g <= 0] == 0)                      # gate closed: no input
    pos = g > 0
    assert np.all(np.sign(t[pos]) == np.sign(u[pos]) * (t[pos] != 0))   # sign of the up branch
    # integer-valued operands small enough to be exact: t is g^2 u exactly
    gi = rng.integers(-20, 21, 5000).astype(np.float32)
    ui = rng.integers(-50, 51, 5000).astype(np.float32)
    ti = orc.relu2_gate(gi, ui)
    want = np.where(gi > 0, gi.astype(np.int64) ** 2 * ui.astype(np.int64), 0)
    assert np.array_equal(ti.astype(np.int64), want)
    # a unit gate passes u through; a power-of-two gate scales u exactly
    assert np.array_equal(orc.relu2_gate(np.ones(100, np.float32), u[:100]), u[:100])
    assert np.array_equal(orc.relu2_gate(np.full(100, 4.0, np.float32), u[:100]), u[:100] * np.float32(16))


def test_relu2_then_quant_equals_quant_of_product(orc):
    """Composition by definition: quantising the gate output is quantising t."""
    rng = np.random.default_rng(8)
    g = rng.standard_normal((3, 256)).astype(np.float32)
    u = rng.standard_normal((3, 256)).astype(np.float32)
    t = orc.relu2_gate(g, u)
    xq, sc, xs = orc.quant_act(t)
    # at least one code of every row with a nonzero input is +-127
    for m in range(3):
        if np.any(t[m] != 0):
            assert np.max(np.abs(xq[m])) == 127
    assert np.array_equal(xs, xq.astype(np.int64).sum(axis=1))


def test_output_resid(orc):
    acc = np.array([[3, -2, 0]], np.int32)
    scale = np.array([2.0], np.float32)
    resid = np.array([[1.0, 0.5, -7.25]], np.float32)
    y = orc.output_resid(acc, 0.5, scale, resid)
    # gamma * s = 1: y = resid + acc exactly
    assert np.array_equal(y, np.array([[4.0, -1.5, -7.25]], np.float32))
    rng = np.random.default_rng(9)
    acc = rng.integers(-100000, 100000, (4, 64)).astype(np.int32)
    scale = rng.random(4).astype(np.float32) * 0.01
    zero = np.zeros((4, 64), np.float32)
    # zero residual: the plain output; zero accumulator: the residual itself
    assert np.array_equal(orc.output_resid(acc, 0.0173, scale, zero), orc.output(acc, 0.0173, scale))
    r = rng.standard_normal((4, 64)).astype(np.float32)
    assert np.array_equal(orc.output_resid(np.zeros_like(acc), 0.0173, scale, r), r)
    # one rounding per operation: product rounded, then the sum
    prod = orc.output(acc, 0.0173, scale)
    assert np.array_equal(orc.output_resid(acc, 0.0173, scale, r), (r + prod).astype(np.float32))


# ---------------------------------------------------------------------------
# BitNet b1 binary weights ("BitNet / Ternary / Binary", BitNet b1 (binaire):
# every weight exactly +1 or -1).
# ---------------------------------------------------------------------------
def test_binarise_sign_rule(orc):
    W = np.array([[0.3, -0.3, 0.0, -0.0, 1e-30, -1e-30, np.nan, np.inf, -np.inf, 5.0, -2.0, 7.0]], np.float32)
    want = np.array([[1, -1, 1, 1, 1, -1, -1, 1, -1, 1, -1, 1]], np.int8)
    assert np.array_equal(orc.binarise(W), want)


def test_binarise_scale_and_idempotence(orc):
    rng = np.random.default_rng(21)
    B = np.where(rng.random((64, 96)) < 0.5, -1, 1).astype(np.int8)
    for c in (0.02, 3.0, 2.0 ** -20):
        W = (B.astype(np.float32) * np.float32(c)).astype(np.float32)
        Wb, beta = orc.quant_weights_b1(W)
        assert np.array_equal(Wb, B)                 # signs of a scaled binary matrix come back
        assert beta == np.float32(c)                 # mean of equal magnitudes is that magnitude
    # beta is the absmean of the latent weights (the ternary gamma statistic)
    W = rng.standard_normal((37, 64)).astype(np.float32)
    assert orc.quant_weights_b1(W)[1] == orc.gamma(W)


def test_pack_b1_golden(orc):
    lines = golden_lines("pack_b1_layout.txt")
    w = np.array([[int(v) for v in lines[0].split()]], np.int8)
    want = np.array([[int(v, 16) for v in lines[1].split()]], np.uint8)
    packed, bad = orc.pack_b1(w)
    assert bad == 0 and np.array_equal(packed, want)


def test_pack_b1_bijection(orc):
    rng = np.random.default_rng(22)
    B = np.where(rng.random((16, 256)) < 0.5, -1, 1).astype(np.int8)
    P, bad = orc.pack_b1(B)
    assert bad == 0 and P.shape == (16, 32)
    assert np.array_equal(orc.unpack_b1(P, 256), B)
    # every byte pattern is a valid packing: unpack then pack is the identity
    R = rng.integers(0, 256, (8, 64), dtype=np.uint8)
    assert np.array_equal(orc.pack_b1(orc.unpack_b1(R, 512))[0], R)
    # each single bit maps to one weight: k = 32g + 4s + j <-> bit 8j + s
    for bit in range(32):
        word = np.array([[bit < 8 and 1 << bit or 0, bit >= 8 and bit < 16 and 1 << (bit - 8) or 0,
                          bit >= 16 and bit < 24 and 1 << (bit - 16) or 0, bit >= 24 and 1 << (bit - 24) or 0]],
                        np.uint8)
        w = orc.unpack_b1(word, 32)[0]
        j, s = bit // 8, bit % 8
        assert np.flatnonzero(w == 1).tolist() == [4 * s + j]
    assert orc.pack_b1(np.zeros((1, 32), np.int8))[1] == 32       # non +-1 values counted


def test_binary_contraction_add_subtract(orc):
    """acc = sum over +1 weights minus sum over -1 weights = 2 * sum_{b=1} x - sum x."""
    rng = np.random.default_rng(23)
    xq = rng.integers(-127, 128, (5, 128)).astype(np.int8)
    B = np.where(rng.random((9, 128)) < 0.5, -1, 1).astype(np.int8)
    acc = orc.linear_i32(xq, B)
    x = xq.astype(np.int64)
    plus = (B == 1).astype(np.int64)
    assert np.array_equal(acc, x @ plus.T - x @ (1 - plus).T)
    assert np.array_equal(acc, 2 * (x @ plus.T) - x.sum(axis=1, keepdims=True))


# ---------------------------------------------------------------------------
# Base-3 packing (five ternary weights per byte, about 1.6 bits per weight:
# "BitNET Family", Memory Efficiency; Hacker News, "2 bits instead of 1.58").
# ---------------------------------------------------------------------------
def test_pack_t3_golden(orc):
    lines = golden_lines("pack_t3_layout.txt")
    w = np.array([[int(v) for v in lines[0].split()]], np.int8)
    want = np.array([[int(v, 16) for v in lines[1].split()]], np.uint8)
    packed, bad = orc.pack_t3(w)
    assert bad == 0 and np.array_equal(packed, want)


@pytest.mark.parametrize("K", [16, 20, 80, 100, 2560, 6912])
def test_pack_t3_roundtrip_and_size(orc, K):
    rng = np.random.default_rng(K)
    q = rng.integers(-1, 2, (7, K)).astype(np.int8)
    P, bad = orc.pack_t3(q)
    assert bad == 0 and P.shape == (7, (K + 79) // 80 * 16)
    back, bad2 = orc.unpack_t3(P, K)
    assert bad2 == 0 and np.array_equal(back, q)
    assert P.max() <= 242
    if K % 80 == 0:
        assert P.shape[1] * 5 == K // 4 * 4        # 20% fewer bytes than 2 bits per weight


def test_pack_t3_every_byte_value(orc):
    """Each of the 243 byte values is one 5-digit base-3 word: digit i of byte j is weight 4i + j."""
    for v in range(256):
        P = np.full((1, 16), 121, np.uint8)          # 121 = every code 1 (weight 0)
        P[0, 0] = v
        w, bad = orc.unpack_t3(P, 80)
        if v <= 242:
            assert bad == 0
            assert [int(w[0, 4 * i]) for i in range(5)] == [(v // 3 ** i) % 3 - 1 for i in range(5)]
            assert orc.pack_t3(w)[0][0, 0] == v
        else:
            assert bad == 1 and all(w[0, 4 * i] == 0 for i in range(5))
    assert orc.pack_t3(np.full((1, 20), 2, np.int8))[1] == 20      # out-of-range values counted
