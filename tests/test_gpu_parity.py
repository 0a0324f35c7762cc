"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.  Integer stages (gamma, W_q, packed bytes, x_q, x_sum,
int32 accumulators) must be bit-exact; outputs must agree within 1e-3
relative (binary32) and 1e-2 relative (bfloat16)."""
import numpy as np
import pytest
import torch

import oracle
import bitlinear_bitnet_linear_b200 as bn
from bitlinear_bitnet_linear_b200 import synthetic

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

DEV = "cuda:0"
RTOL = {torch.float32: 1e-3, torch.bfloat16: 1e-2}


@pytest.fixture(scope="module", autouse=True)
def _built():
    from bitlinear_bitnet_linear_b200 import build
    build.build()
    oracle.build()
    torch.cuda.set_device(0)


def to_np(t):
    return t.detach().cpu().numpy()


def xf32(x):
    """bfloat16 -> binary32 widening (exact), as numpy."""
    return x.float().numpy()


def assert_y(y_gpu, y_ref, dtype):
    a = y_gpu.float().cpu().numpy().astype(np.float64)
    b = y_ref.astype(np.float64)
    err = np.abs(a - b)
    bound = RTOL[dtype] * np.abs(b)
    bad = err > bound
    assert not bad.any(), (f"{bad.sum()} of {bad.size} outside rtol {RTOL[dtype]}; "
                           f"worst rel {(err / np.maximum(np.abs(b), 1e-30)).max():.3e}")


# ---------------------------------------------------------------------------
# weight preparation
# ---------------------------------------------------------------------------

WEIGHT_SHAPES = [(256, 256, 0), (1, 16, 1), (257, 272, 2), (2560, 2560, 3), (6912, 2560, 4), (2560, 6912, 5)]


@pytest.mark.parametrize("N,K,seed", WEIGHT_SHAPES)
def test_quant_weights_bitexact(N, K, seed):
    W = synthetic.latent_weights(N, K, seed)
    Wq_ref, g_ref = oracle.quant_weights(W.numpy())
    Wq, g = bn.bitnet_quant_weights(W.to(DEV))
    assert to_np(g)[0] == g_ref                      # exact summation: bit-exact gamma
    assert (to_np(Wq) == Wq_ref).all()


def test_quant_weights_wide_range_exact_sum():
    """Subnormals, huge and tiny magnitudes: the exact sum still matches."""
    rng = np.random.default_rng(0)
    e = rng.integers(-149, 100, 64 * 1024)
    v = ((rng.random(e.size) + 0.5) * np.exp2(e.astype(np.float64))).astype(np.float32)
    v *= np.where(rng.random(e.size) < 0.5, -1, 1).astype(np.float32)
    W = torch.from_numpy(v.reshape(256, 256))
    g_ref = oracle.gamma(W.numpy())
    _, g = bn.bitnet_quant_weights(W.to(DEV))
    assert to_np(g)[0] == g_ref


def test_quant_weights_full_70b_shape():
    """8192 x 28672 (the 70B-class FFN up shape): gamma and W_q bit-exact."""
    W = synthetic.latent_weights(28672, 8192, seed=77)
    Wq_ref, g_ref = oracle.quant_weights(W.numpy())
    Wq, g = bn.bitnet_quant_weights(W.to(DEV))
    assert to_np(g)[0] == g_ref
    assert torch.equal(Wq.cpu(), torch.from_numpy(Wq_ref))


def test_ternarise_with_given_gamma_and_ties():
    """gamma = 1 makes W/(gamma+eps) = W: half-way values pin ties-to-even."""
    W = torch.tensor([[0.5, -0.5, 1.5, -1.5, 2.5, -2.5, 0.49999997, 0.50000006] * 2], dtype=torch.float32)
    g = torch.ones(1, dtype=torch.float32, device=DEV)
    Wq = bn.bitnet_ternarise(W.to(DEV), g)
    assert (to_np(Wq) == oracle.ternarise(W.numpy(), np.float32(1.0))).all()
    assert to_np(Wq)[0, :8].tolist() == [0, 0, 1, -1, 1, -1, 0, 1]


def test_quant_weights_degenerate():
    W = torch.zeros((16, 32), dtype=torch.float32)
    Wq, g = bn.bitnet_quant_weights(W.to(DEV))
    assert to_np(g)[0] == 0.0 and (to_np(Wq) == 0).all()
    W = torch.full((3, 16), -2.0)
    Wq, g = bn.bitnet_quant_weights(W.to(DEV))
    assert to_np(g)[0] == 2.0 and (to_np(Wq) == -1).all()


@pytest.mark.parametrize("N,K", [(1, 16), (3, 48), (257, 272), (2560, 6912)])
def test_pack_bitexact_and_roundtrip(N, K):
    rng = np.random.default_rng(N + K)
    q = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    ref, bad = oracle.pack(q)
    Wp = bn.bitnet_pack(torch.from_numpy(q).to(DEV))
    assert (to_np(Wp) == ref).all()
    back = bn.bitnet_unpack(Wp, K)
    assert (to_np(back) == q).all()


def test_pack_invalid_values_counted():
    q = np.zeros((2, 32), np.int8)
    q[0, 5] = 3
    q[1, 31] = -2
    cnt = torch.zeros(1, dtype=torch.int32, device=DEV)
    Wp = bn.bitnet_pack(torch.from_numpy(q).to(DEV), n_invalid=cnt)
    ref, bad = oracle.pack(q)
    assert (to_np(Wp) == ref).all() and int(cnt.item()) == bad == 2
    cnt2 = torch.zeros(1, dtype=torch.int32, device=DEV)
    back = bn.bitnet_unpack(Wp, 32, n_invalid=cnt2)
    ref_back, bad2 = oracle.unpack(ref, 32)
    assert int(cnt2.item()) == bad2 == 2 and (to_np(back) == ref_back).all()


# ---------------------------------------------------------------------------
# activation quantisation
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("M,K", [(1, 16), (3, 272), (7, 2560), (65, 6912), (4096, 2560)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("norm", [False, True])
def test_quant_act(M, K, dtype, norm):
    x = synthetic.activations(M, K, seed=M * 7 + K, dtype=dtype)
    gain = None
    if norm:
        gain = torch.from_numpy(np.random.default_rng(K).uniform(0.5, 1.5, K).astype(np.float32))
    xq_ref, sc_ref, xs_ref = oracle.quant_act(xf32(x), None if gain is None else gain.numpy(), 1e-5)
    xq, sc, xs = bn.bitnet_quant_act(x.to(DEV), None if gain is None else gain.to(DEV), 1e-5)
    assert (to_np(xq) == xq_ref).all()
    assert (to_np(xs) == xs_ref).all()
    if norm:
        assert np.allclose(to_np(sc), sc_ref, rtol=1e-6, atol=0)
    else:
        assert (to_np(sc) == sc_ref).all()


def test_quant_act_zero_and_tiny_rows():
    x = torch.zeros((3, 64), dtype=torch.float32)
    x[1, 3] = 1e-7
    x[2, :] = 1e-30
    xq_ref, sc_ref, xs_ref = oracle.quant_act(x.numpy())
    xq, sc, xs = bn.bitnet_quant_act(x.to(DEV))
    assert (to_np(xq) == xq_ref).all() and (to_np(sc) == sc_ref).all() and (to_np(xs) == xs_ref).all()


# ---------------------------------------------------------------------------
# contraction: exact int32 accumulators on both paths
# ---------------------------------------------------------------------------

def _prep(M, K, N, seed, xdtype=torch.bfloat16):
    W = synthetic.latent_weights(N, K, seed)
    Wq, g = oracle.quant_weights(W.numpy())
    Wp, _ = oracle.pack(Wq)
    x = synthetic.activations(M, K, seed + 1, dtype=xdtype)
    return W, Wq, g, Wp, x


ACC_CASES = [
    (1, 256, 256), (1, 2560, 2560), (2, 2560, 6912), (3, 272, 257), (4, 6912, 2560), (4, 336, 1),
    (1, 16, 5), (5, 2560, 300), (16, 128, 128), (17, 272, 129), (64, 2560, 6912), (100, 336, 129),
    (129, 1024, 1000), (257, 2560, 384), (300, 64, 200),
    # 512 tokens and more: tiles of 128 weight rows x 256 tokens, ragged in both
    (512, 256, 128), (600, 1024, 1000), (777, 272, 129),
    # the persistent kernel's edges: one token over the small-kernel limit, a
    # single weight row, K below one 128-wide block (scalar weight loads)
    (65, 2560, 7), (70, 16, 1), (1000, 32, 2),
]


@pytest.mark.parametrize("M,K,N", ACC_CASES)
def test_accumulator_bitexact(M, K, N):
    _, Wq, g, Wp, x = _prep(M, K, N, seed=M + K + N)
    xq_ref, sc_ref, xs_ref = oracle.quant_act(xf32(x))
    acc_ref = oracle.linear_i32(xq_ref, Wq)
    xq = torch.from_numpy(xq_ref).to(DEV)
    sc = torch.from_numpy(sc_ref).to(DEV)
    Wp_d = torch.from_numpy(Wp).to(DEV)
    gd = torch.tensor([g], dtype=torch.float32, device=DEV)
    paths = [bn.PATH_TC] + ([bn.PATH_GEMV] if M <= 4 else [])
    for path in paths:
        for xs_in in (None, torch.from_numpy(xs_ref).to(DEV)):
            _, acc = bn.bitnet_linear_q(xq, sc, Wp_d, gd, x_sum=xs_in, want_y=False, want_acc=True, path=path)
            torch.cuda.synchronize()
            got = to_np(acc)
            assert (got == acc_ref).all(), f"path {path}: {(got != acc_ref).sum()} mismatches"


# ---------------------------------------------------------------------------
# end to end: x -> y
# ---------------------------------------------------------------------------

E2E_CASES = [
    # (M, K, N, x dtype, y dtype, gain)
    (1, 256, 256, torch.float32, torch.float32, False),     # single BitLinear, fp32 in/out
    (1, 2560, 2560, torch.bfloat16, torch.bfloat16, False),
    (1, 2560, 6912, torch.bfloat16, torch.bfloat16, False),
    (1, 6912, 2560, torch.bfloat16, torch.bfloat16, False),
    (4, 2560, 6912, torch.bfloat16, torch.bfloat16, True),
    (3, 272, 257, torch.float32, torch.float32, True),
    (16, 2560, 6912, torch.bfloat16, torch.bfloat16, True),
    (64, 2560, 6912, torch.bfloat16, torch.bfloat16, True),
    (200, 336, 130, torch.float32, torch.bfloat16, False),
    (700, 336, 130, torch.float32, torch.bfloat16, False),
    (530, 2560, 1000, torch.bfloat16, torch.float32, True),
]


@pytest.mark.parametrize("M,K,N,xd,yd,norm", E2E_CASES)
def test_linear_end_to_end(M, K, N, xd, yd, norm):
    W, Wq, g, Wp, x = _prep(M, K, N, seed=3 * M + K, xdtype=xd)
    gain = synthetic.unit_gain(K) if norm else None
    y_ref, *_ = oracle.bitlinear(xf32(x), Wq, g, None if gain is None else gain.numpy(), 1e-5)
    # the whole GPU chain: quantise and pack the weights on the device too
    Wq_d, g_d = bn.bitnet_quant_weights(W.to(DEV))
    Wp_d = bn.bitnet_pack(Wq_d)
    assert (to_np(Wp_d) == Wp).all()
    paths = [bn.PATH_AUTO, bn.PATH_TC] + ([bn.PATH_GEMV] if M <= 4 else [])
    for path in paths:
        y = bn.bitnet_linear(x.to(DEV), Wp_d, g_d, rms_gain=None if gain is None else gain.to(DEV),
                             y_dtype=yd, path=path)
        torch.cuda.synchronize()
        assert_y(y, y_ref, yd)
        if not norm:
            # without the norm every float step is a fixed sequence of IEEE ops: bit-exact
            ref = y_ref if yd == torch.float32 else oracle.to_bf16_bits(y_ref)
            got = to_np(y) if yd == torch.float32 else to_np(y.view(torch.int16)).view(np.uint16)
            assert (got == ref).all()


# ---------------------------------------------------------------------------
# full-size configurations, sampled rows checked against the oracle
# ---------------------------------------------------------------------------

def _sampled_check(M, K, N, seed, norm, sample_rows):
    W, Wq, g, Wp, x = _prep(M, K, N, seed)
    gain = synthetic.unit_gain(K) if norm else None
    Wp_d = torch.from_numpy(Wp).to(DEV)
    gd = torch.tensor([g], dtype=torch.float32, device=DEV)
    y = bn.bitnet_linear(x.to(DEV), Wp_d, gd, rms_gain=None if gain is None else gain.to(DEV),
                         y_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    rows = sorted(set([0, M - 1] + list(np.random.default_rng(seed).integers(0, M, sample_rows))))
    xs = xf32(x)[rows]
    y_ref, *_ = oracle.bitlinear(xs, Wq, g, None if gain is None else gain.numpy(), 1e-5)
    assert_y(y[rows], y_ref, torch.bfloat16)
    assert torch.isfinite(y.float()).all()


@pytest.mark.parametrize("M", [1, 4, 16, 64, 256, 1024, 4096])
def test_sweep_k2560_n6912_sampled(M):
    _sampled_check(M, 2560, 6912, seed=500 + M, norm=True, sample_rows=6)


@pytest.mark.parametrize("M", [1, 8, 512])
@pytest.mark.parametrize("K,N", [(8192, 28672), (28672, 8192)])
def test_large_shapes_sampled(M, K, N):
    _sampled_check(M, K, N, seed=900 + M + K, norm=False, sample_rows=2)


# K beyond the fused GEMV's shared-memory bound (48128 at M = 1, 39936 at
# M = 2, 29696 at M = 3, 4): the automatic path takes the tensor-core GEMM,
# the forced GEMV path reports UNSUPPORTED
@pytest.mark.parametrize("M,K", [(1, 53248), (1, 57344), (2, 45056), (4, 32768)])
def test_long_rows_take_tensor_core_path(M, K):
    N = 40
    _, Wq, g, Wp, x = _prep(M, K, N, seed=M + K)
    y_ref, *_ = oracle.bitlinear(xf32(x), Wq, g)
    Wp_d = torch.from_numpy(Wp).to(DEV)
    gd = torch.tensor([g], dtype=torch.float32, device=DEV)
    y = bn.bitnet_linear(x.to(DEV), Wp_d, gd, y_dtype=torch.float32)
    torch.cuda.synchronize()
    assert np.array_equal(to_np(y), y_ref)   # no gain: the same IEEE operations, bit-exact
    with pytest.raises(bn.BitnetError) as ei:
        bn.bitnet_linear(x.to(DEV), Wp_d, gd, path=bn.PATH_GEMV)
    assert ei.value.status == 5


# ---------------------------------------------------------------------------
# errors and the watchdog
# ---------------------------------------------------------------------------

def test_forced_gemv_rejects_large_m():
    _, _, g, Wp, x = _prep(8, 256, 64, seed=1)
    with pytest.raises(bn.BitnetError) as ei:
        bn.bitnet_linear(x.to(DEV), torch.from_numpy(Wp).to(DEV), torch.tensor([g], device=DEV),
                         path=bn.PATH_GEMV)
    assert ei.value.status == 5


def test_workspace_too_small():
    _, _, g, Wp, x = _prep(64, 256, 64, seed=2)
    ws = bn.new_workspace(256)
    with pytest.raises(bn.BitnetError) as ei:
        bn.bitnet_linear(x.to(DEV), torch.from_numpy(Wp).to(DEV), torch.tensor([g], device=DEV), ws=ws)
    assert ei.value.status == 8


def test_watchdog_records_timeout_and_context_survives():
    ws = bn.new_workspace(256)
    bn.bitnet_watchdog_selftest(ws, 2000)          # 2 ms wait on a barrier nobody completes
    assert bn.bitnet_get_error(ws) == 7
    assert bn.bitnet_get_error(ws) == 0            # cleared after reading
    # the context is still usable
    _, Wq, g, Wp, x = _prep(1, 256, 256, seed=3)
    y = bn.bitnet_linear(x.to(DEV), torch.from_numpy(Wp).to(DEV), torch.tensor([g], device=DEV))
    torch.cuda.synchronize()
    y_ref, *_ = oracle.bitlinear(xf32(x), Wq, g)
    assert_y(y, y_ref, torch.bfloat16)


def test_no_device_errors_after_suite():
    ws = bn.new_workspace(bn.bitnet_workspace_bytes(300, 2560, 512))
    _, _, g, Wp, x = _prep(300, 2560, 512, seed=4)
    bn.bitnet_linear(x.to(DEV), torch.from_numpy(Wp).to(DEV), torch.tensor([g], device=DEV), ws=ws)
    assert bn.bitnet_get_error(ws) == 0


# ---------------------------------------------------------------------------
# grouped GEMV: many problems in one launch
# ---------------------------------------------------------------------------

def _grouped_case(specs, M, xd, yd, norm, seed):
    """specs: list of (K, N, share_x_with_previous)."""
    problems, refs = [], []
    x = x_np = None
    for i, (K, N, share) in enumerate(specs):
        W = synthetic.latent_weights(N, K, seed + 17 * i)
        Wq, g = oracle.quant_weights(W.numpy())
        Wp, _ = oracle.pack(Wq)
        if not share:
            x = synthetic.activations(M, K, seed + 31 * i, dtype=xd)
            x_np = xf32(x)
            x_dev = x.to(DEV)
            gain = (torch.from_numpy(np.random.default_rng(seed + i).uniform(0.5, 1.5, K).astype(np.float32))
                    if norm else None)
            gain_dev = None if gain is None else gain.to(DEV)
        y = torch.empty((M, N), dtype=yd, device=DEV)
        problems.append((x_dev, torch.from_numpy(Wp).to(DEV), torch.tensor([g], dtype=torch.float32, device=DEV),
                         gain_dev, y))
        y_ref, *_ = oracle.bitlinear(x_np, Wq, g, None if gain is None else gain.numpy(), 1e-5)
        refs.append(y_ref)
    return problems, refs


@pytest.mark.parametrize("M", [1, 2, 3, 4])
@pytest.mark.parametrize("norm", [False, True])
def test_grouped_small_mixed(M, norm):
    specs = [(2560, 256, False), (2560, 256, True), (2560, 384, True), (6912, 128, False), (256, 64, False),
             (2560, 300, False)]
    problems, refs = _grouped_case(specs, M, torch.bfloat16, torch.bfloat16, norm, seed=40 + M)
    ws = bn.new_workspace(256)
    bn.bitnet_linear_grouped(problems, ws=ws)
    assert bn.bitnet_get_error(ws) == 0
    for (x, Wp, g, gain, y), y_ref in zip(problems, refs):
        assert_y(y, y_ref, torch.bfloat16)
        if not norm:
            assert (to_np(y.view(torch.int16)).view(np.uint16) == oracle.to_bf16_bits(y_ref)).all()


def test_grouped_stack_layer_deep_ring():
    """One transformer block's seven calls twice (> 32 MB of weights: the
    deep-ring, one-CTA-per-SM configuration), fp32 in and out."""
    layer = [(2560, 2560, False), (2560, 2560, True), (2560, 2560, True), (2560, 2560, False),
             (2560, 6912, False), (2560, 6912, True), (6912, 2560, False)]
    problems, refs = _grouped_case(layer * 2, 1, torch.float32, torch.float32, False, seed=77)
    ws = bn.new_workspace(256)
    bn.bitnet_linear_grouped(problems, ws=ws)
    assert bn.bitnet_get_error(ws) == 0
    for (x, Wp, g, gain, y), y_ref in zip(problems, refs):
        assert (to_np(y) == y_ref).all()


def test_grouped_rejects_bad_arguments():
    x = torch.zeros((1, 96), dtype=torch.bfloat16, device=DEV)      # K % 64 != 0
    Wp = torch.zeros((8, 24), dtype=torch.uint8, device=DEV)
    y = torch.zeros((1, 8), dtype=torch.bfloat16, device=DEV)
    g = torch.ones(1, device=DEV)
    with pytest.raises(bn.BitnetError) as ei:
        bn.bitnet_linear_grouped([(x, Wp, g, None, y)])
    assert ei.value.status == 2
    x5 = torch.zeros((5, 128), dtype=torch.bfloat16, device=DEV)     # M > 4
    with pytest.raises(bn.BitnetError):
        bn.bitnet_linear_grouped([(x5, torch.zeros((8, 32), dtype=torch.uint8, device=DEV), g, None,
                                   torch.zeros((5, 8), dtype=torch.bfloat16, device=DEV))])
