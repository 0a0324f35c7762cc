"""GPU parity of the BitNet b1 binary-weight path ("BitNet / Ternary /
Binary", BitNet b1 (binaire): weights exactly +1 or -1) against the oracle:
beta and the signs bit-exact, the 1-bit packing bit-exact, and the forward
bit-exact in binary32 and in bfloat16 (same operations in the same order)."""
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


@pytest.mark.parametrize("N,K,seed", [(256, 256, 0), (2560, 2560, 1), (6912, 2560, 2), (2560, 6912, 3), (3, 32, 4)])
def test_quant_weights_b1_bitexact(N, K, seed):
    W = synthetic.latent_weights(N, K, seed)
    Wb_ref, beta_ref = oracle.quant_weights_b1(W.numpy())
    Wb, beta = bn.bitnet_quant_weights_b1(W.to(DEV))
    assert beta.cpu().numpy()[0] == beta_ref
    assert np.array_equal(Wb.cpu().numpy(), Wb_ref)


def test_binarise_special_values():
    W = torch.tensor([[0.0, -0.0, 1e-30, -1e-30, 2.0, -2.0, 1e-3, -1e-3] * 4], dtype=torch.float32)
    Wb, _ = bn.bitnet_quant_weights_b1(W.to(DEV))
    assert np.array_equal(Wb.cpu().numpy(), oracle.binarise(W.numpy()))


@pytest.mark.parametrize("N,K", [(1, 32), (77, 256), (2560, 6912)])
def test_pack_b1_bitexact_and_roundtrip(N, K):
    rng = np.random.default_rng(N + K)
    Wb = np.where(rng.random((N, K)) < 0.5, -1, 1).astype(np.int8)
    ref, bad = oracle.pack_b1(Wb)
    assert bad == 0
    Wp = bn.bitnet_pack_b1(torch.from_numpy(Wb).to(DEV))
    assert np.array_equal(Wp.cpu().numpy(), ref)
    assert np.array_equal(bn.bitnet_unpack_b1(Wp, K).cpu().numpy(), Wb)


def test_pack_b1_counts_invalid():
    Wb = np.ones((4, 64), np.int8)
    Wb[0, 3] = 0
    Wb[2, 40] = 5
    cnt = torch.zeros(1, dtype=torch.int32, device=DEV)
    Wp = bn.bitnet_pack_b1(torch.from_numpy(Wb).to(DEV), n_invalid=cnt)
    ref, bad = oracle.pack_b1(Wb)
    torch.cuda.synchronize()
    assert int(cnt.item()) == bad == 2
    assert np.array_equal(Wp.cpu().numpy(), ref)


def b1_weights(N, K, seed):
    W = synthetic.latent_weights(N, K, seed)
    Wb, beta = oracle.quant_weights_b1(W.numpy())
    Wp, _ = oracle.pack_b1(Wb)
    return Wb, beta, torch.from_numpy(Wp).to(DEV), torch.tensor([beta], dtype=torch.float32, device=DEV)


# M = 1: the streaming GEMV (1-bit lane groups); M > 1: the tensor-core path
@pytest.mark.parametrize("M,K,N", [(1, 2560, 2560), (1, 6912, 2560), (1, 2560, 6912), (1, 128, 37),
                                   (1, 8192, 640), (2, 2560, 384), (64, 2560, 1000), (300, 6912, 512),
                                   (5, 384, 130), (600, 2560, 300)])
@pytest.mark.parametrize("with_gain", [False, True])
def test_linear_b1_matches_oracle(M, K, N, with_gain):
    x = synthetic.activations(M, K, seed=500 + M + K, dtype=torch.bfloat16)
    Wb, beta, Wp, beta_d = b1_weights(N, K, seed=600 + N)
    gain = synthetic.unit_gain(K) if with_gain else None
    xq, sc, _ = oracle.quant_act(x.float().numpy(), None if gain is None else gain.numpy())
    y_ref = oracle.output(oracle.linear_i32(xq, Wb), beta, sc)
    g = None if gain is None else gain.to(DEV)
    y32 = bn.bitnet_linear_b1(x.to(DEV), Wp, beta_d, N=N, rms_gain=g, y_dtype=torch.float32)
    y16 = bn.bitnet_linear_b1(x.to(DEV), Wp, beta_d, N=N, rms_gain=g, y_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert np.array_equal(y32.cpu().numpy(), y_ref)
    assert np.array_equal(y16.cpu().view(torch.int16).numpy().astype(np.uint16), oracle.to_bf16_bits(y_ref))


def test_linear_b1_long_row_takes_tensor_core_path():
    """M = 1 with K beyond the fused GEMV's bound for 1-bit rows (79872)."""
    M, K, N = 1, 81920, 24
    x = synthetic.activations(M, K, seed=321, dtype=torch.bfloat16)
    Wb, beta, Wp, beta_d = b1_weights(N, K, seed=654)
    xq, sc, _ = oracle.quant_act(x.float().numpy())
    y_ref = oracle.output(oracle.linear_i32(xq, Wb), beta, sc)
    y = bn.bitnet_linear_b1(x.to(DEV), Wp, beta_d, N=N, y_dtype=torch.float32)
    torch.cuda.synchronize()
    assert np.array_equal(y.cpu().numpy(), y_ref)


def test_linear_b1_rejects_k_not_multiple_of_128():
    x = torch.zeros(1, 192, dtype=torch.bfloat16, device=DEV)
    Wp = torch.zeros(8, 24, dtype=torch.uint8, device=DEV)
    beta = torch.ones(1, device=DEV)
    with pytest.raises(bn.BitnetError, match="SHAPE"):
        bn.bitnet_linear_b1(x, Wp, beta)


def test_grouped_b1_matches_single_calls():
    shapes = [(2560, 2560), (2560, 6912), (6912, 2560), (128, 45)]
    probs, refs = [], []
    gain = {K: synthetic.unit_gain(K).to(DEV) for K, _ in shapes}
    for i, (K, N) in enumerate(shapes):
        x = synthetic.activations(1, K, seed=700 + i, dtype=torch.bfloat16)
        Wb, beta, Wp, beta_d = b1_weights(N, K, seed=800 + i)
        xq, sc, _ = oracle.quant_act(x.float().numpy(), synthetic.unit_gain(K).numpy())
        refs.append(oracle.output(oracle.linear_i32(xq, Wb), beta, sc))
        y = torch.empty(1, N, dtype=torch.float32, device=DEV)
        probs.append((x.to(DEV), Wp, beta_d, gain[K], y))
    call = bn.GroupedCall(probs, bits=1)
    call()
    torch.cuda.synchronize()
    for (_, _, _, _, y), ref in zip(probs, refs):
        assert np.array_equal(y.cpu().numpy(), ref)
