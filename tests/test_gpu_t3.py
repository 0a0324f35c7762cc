"""GPU parity of base-3 packing (five ternary weights per byte, about 1.6
bits per weight: "BitNET Family", Memory Efficiency) against the oracle:
packed bytes bit-exact, and the one-token forward bit-exact in binary32 and
bfloat16 against the oracle's ternary forward (the format only changes how
the same ternary weights are stored)."""
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


def ternary(N, K, seed):
    W = synthetic.latent_weights(N, K, seed)
    return oracle.quant_weights(W.numpy())


@pytest.mark.parametrize("N,K", [(1, 16), (33, 112), (256, 2560), (2560, 6912)])
def test_pack_t3_bitexact_and_roundtrip(N, K):
    Wq, _ = ternary(N, K, seed=N + K)
    ref, bad = oracle.pack_t3(Wq)
    assert bad == 0
    assert bn.bitnet_t3_row_bytes(K) == ref.shape[1]
    Wp = bn.bitnet_pack_t3(torch.from_numpy(Wq).to(DEV))
    assert np.array_equal(Wp.cpu().numpy(), ref)
    assert np.array_equal(bn.bitnet_unpack_t3(Wp, K).cpu().numpy(), Wq)


def test_t3_invalid_values_counted():
    Wq = np.zeros((2, 48), np.int8)
    Wq[0, 7] = 2
    Wq[1, 39] = -5
    cnt = torch.zeros(1, dtype=torch.int32, device=DEV)
    Wp = bn.bitnet_pack_t3(torch.from_numpy(Wq).to(DEV), n_invalid=cnt)
    ref, bad = oracle.pack_t3(Wq)
    torch.cuda.synchronize()
    assert int(cnt.item()) == bad == 2 and np.array_equal(Wp.cpu().numpy(), ref)
    raw = torch.full((1, 16), 250, dtype=torch.uint8, device=DEV)       # every byte above 242
    cnt.zero_()
    w = bn.bitnet_unpack_t3(raw, 80, n_invalid=cnt)
    torch.cuda.synchronize()
    ref_w, bad_w = oracle.unpack_t3(raw.cpu().numpy(), 80)
    assert int(cnt.item()) == bad_w and np.array_equal(w.cpu().numpy(), ref_w)


@pytest.mark.parametrize("K,N", [(2560, 2560), (2560, 6912), (6912, 2560), (112, 77), (16, 5), (8192, 1024),
                                 (28672, 256)])
@pytest.mark.parametrize("with_gain", [False, True])
def test_linear_t3_matches_oracle(K, N, with_gain):
    x = synthetic.activations(1, K, seed=900 + K, dtype=torch.bfloat16)
    Wq, gam = ternary(N, K, seed=1000 + N)
    Wp = torch.from_numpy(oracle.pack_t3(Wq)[0]).to(DEV)
    gam_d = torch.tensor([gam], dtype=torch.float32, device=DEV)
    gain = synthetic.unit_gain(K) if with_gain else None
    xq, sc, _ = oracle.quant_act(x.float().numpy(), None if gain is None else gain.numpy())
    y_ref = oracle.output(oracle.linear_i32(xq, Wq), gam, sc)
    g = None if gain is None else gain.to(DEV)
    y32 = bn.bitnet_linear_t3(x.to(DEV), Wp, gam_d, N=N, rms_gain=g, y_dtype=torch.float32)
    y16 = bn.bitnet_linear_t3(x.to(DEV), Wp, gam_d, N=N, rms_gain=g, y_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert np.array_equal(y32.cpu().numpy(), y_ref)
    assert np.array_equal(y16.cpu().view(torch.int16).numpy().astype(np.uint16), oracle.to_bf16_bits(y_ref))


def test_grouped_t3_matches_oracle():
    shapes = [(2560, 2560), (2560, 6912), (6912, 2560), (112, 45)]
    probs, refs = [], []
    for i, (K, N) in enumerate(shapes):
        x = synthetic.activations(1, K, seed=1100 + i, dtype=torch.bfloat16)
        Wq, gam = ternary(N, K, seed=1200 + i)
        xq, sc, _ = oracle.quant_act(x.float().numpy(), synthetic.unit_gain(K).numpy())
        refs.append(oracle.output(oracle.linear_i32(xq, Wq), gam, sc))
        Wp = torch.from_numpy(oracle.pack_t3(Wq)[0]).to(DEV)
        y = torch.empty(1, N, dtype=torch.float32, device=DEV)
        probs.append((x.to(DEV), Wp, torch.tensor([gam], device=DEV), synthetic.unit_gain(K).to(DEV), y))
    bn.GroupedCall(probs, bits=3)()
    torch.cuda.synchronize()
    for (_, _, _, _, y), ref in zip(probs, refs):
        assert np.array_equal(y.cpu().numpy(), ref)


def test_linear_t3_rejects_more_than_one_token():
    with pytest.raises(ValueError):
        bn.bitnet_linear_t3(torch.zeros(2, 160, dtype=torch.bfloat16, device=DEV),
                            torch.zeros(4, 32, dtype=torch.uint8, device=DEV), torch.ones(1, device=DEV))
