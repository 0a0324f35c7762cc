"""GPU parity of the feed-forward down projection with the ReLU^2 gate fused
into the activation quantiser, and of the optional residual add ("Key
Technologies ...", Architectural Innovations: squared ReLU in the
feed-forward layers).  Codes, scales and code sums are bit-exact against the
oracle; outputs are bit-exact too (same binary32 operations in the same
order), checked also against the stated tolerances."""
import numpy as np
import pytest
import torch

import oracle
import bitlinear_bitnet_linear_b200 as bn
from bitlinear_bitnet_linear_b200 import synthetic

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from bitlinear_bitnet_linear_b200 import build
    build.build()
    oracle.build()
    torch.cuda.set_device(0)


def gate_up(M, K, seed, dtype):
    """Gate and up projection outputs: N(0,1) with 1% outliers x20."""
    g = synthetic.activations(M, K, seed=seed, dtype=dtype)
    u = synthetic.activations(M, K, seed=seed + 1, dtype=dtype)
    return g, u


def ternary(N, K, seed):
    W = synthetic.latent_weights(N, K, seed)
    Wq, g = oracle.quant_weights(W.numpy())
    Wp, _ = oracle.pack(Wq)
    return Wq, g, torch.from_numpy(Wp).to(DEV), torch.tensor([g], dtype=torch.float32, device=DEV)


@pytest.mark.parametrize("M,K", [(1, 6912), (3, 2560), (64, 2560), (5, 272)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("with_gain", [False, True])
def test_quant_act_relu2_bitexact(M, K, dtype, with_gain):
    g, u = gate_up(M, K, seed=100 + M + K, dtype=dtype)
    gain = synthetic.unit_gain(K) if with_gain else None
    t = oracle.relu2_gate(g.float().numpy(), u.float().numpy())
    xq_ref, sc_ref, xs_ref = oracle.quant_act(t, None if gain is None else gain.numpy())
    xq, sc, xs = bn.bitnet_quant_act_relu2(g.to(DEV), u.to(DEV), None if gain is None else gain.to(DEV))
    assert np.array_equal(xq.cpu().numpy(), xq_ref)
    assert np.array_equal(sc.cpu().numpy(), sc_ref)
    assert np.array_equal(xs.cpu().numpy(), xs_ref)


# M <= 4 with K % 64 == 0: the streaming GEMV; otherwise the tensor-core path
@pytest.mark.parametrize("M,K,N", [(1, 6912, 2560), (2, 2560, 1000), (4, 6912, 256), (16, 2560, 384),
                                   (300, 2560, 512), (3, 272, 130), (520, 2560, 200)])
@pytest.mark.parametrize("y_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("with_resid", [False, True])
def test_linear_relu2_matches_oracle(M, K, N, y_dtype, with_resid):
    g, u = gate_up(M, K, seed=200 + M + N, dtype=torch.bfloat16)
    Wq, gam, Wp, gam_d = ternary(N, K, seed=300 + N)
    gain = synthetic.unit_gain(K)
    t = oracle.relu2_gate(g.float().numpy(), u.float().numpy())
    xq, sc, _ = oracle.quant_act(t, gain.numpy())
    acc = oracle.linear_i32(xq, Wq)
    resid = None
    if with_resid:
        resid = synthetic.activations(M, N, seed=400 + N, dtype=y_dtype)
        y_ref = oracle.output_resid(acc, gam, sc, resid.float().numpy())
    else:
        y_ref = oracle.output(acc, gam, sc)
    y = bn.bitnet_linear_relu2(g.to(DEV), u.to(DEV), Wp, gam_d, N=N, rms_gain=gain.to(DEV),
                               resid=None if resid is None else resid.to(DEV), y_dtype=y_dtype)
    torch.cuda.synchronize()
    if y_dtype == torch.float32:
        assert np.array_equal(y.cpu().numpy(), y_ref)
    else:
        got = y.cpu().view(torch.int16).numpy().astype(np.uint16)
        assert np.array_equal(got, oracle.to_bf16_bits(y_ref))


def test_linear_relu2_resid_in_place():
    """resid may alias y: the residual stream updated in place."""
    M, K, N = 1, 6912, 2560
    g, u = gate_up(M, K, seed=11, dtype=torch.bfloat16)
    Wq, gam, Wp, gam_d = ternary(N, K, seed=12)
    h = synthetic.activations(M, N, seed=13, dtype=torch.bfloat16)
    t = oracle.relu2_gate(g.float().numpy(), u.float().numpy())
    xq, sc, _ = oracle.quant_act(t)
    y_ref = oracle.output_resid(oracle.linear_i32(xq, Wq), gam, sc, h.float().numpy())
    hd = h.to(DEV)
    bn.bitnet_linear_relu2(g.to(DEV), u.to(DEV), Wp, gam_d, N=N, resid=hd, y=hd)
    torch.cuda.synchronize()
    assert np.array_equal(hd.cpu().view(torch.int16).numpy().astype(np.uint16), oracle.to_bf16_bits(y_ref))


def test_linear_relu2_rejects_bad_arguments():
    g, u = gate_up(1, 256, seed=1, dtype=torch.bfloat16)
    Wq, gam, Wp, gam_d = ternary(64, 256, seed=2)
    with pytest.raises(ValueError):
        bn.bitnet_linear_relu2(g.to(DEV), u.float().to(DEV), Wp, gam_d)
    with pytest.raises(ValueError):
        bn.bitnet_linear_relu2(g.to(DEV), u.to(DEV), Wp, gam_d,
                               resid=torch.zeros(1, 63, dtype=torch.bfloat16, device=DEV))
