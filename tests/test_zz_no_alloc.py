"""bitnet_quant_weights_noalloc: the weight-quantisation entry point that
uses the library's own scratch array instead of a caller workspace.

Its results must equal bitnet_quant_weights' (gamma and W_q bit-exact, the
bar the other weight-stage tests use), on consecutive calls that reuse the
shared scratch with different shapes."""
import ctypes

import pytest
import torch

from bitlinear_bitnet_linear_b200 import _binding as B
from bitlinear_bitnet_linear_b200 import synthetic


def test_noalloc_rejects_beyond_scratch_limit():
    """N*K above 2048 * 2^24 returns BITNET_ERR_SHAPE before any device work
    (the size check precedes the device query, so this runs without a GPU)."""
    buf = (ctypes.c_float * 32)()
    addr = (ctypes.addressof(buf) + 15) // 16 * 16   # 16-byte aligned, never dereferenced
    gamma = ctypes.c_float()
    lib = B.lib()
    N, K = 2048 * 1024 + 1, 16 * 1024   # N*K = 2^35 + 16384 > 2048 * 2^24
    st = lib.bitnet_quant_weights_noalloc(ctypes.c_void_p(addr), N, K, 1e-8, None,
                                          ctypes.byref(gamma), None)
    assert st == 2   # BITNET_ERR_SHAPE
    with pytest.raises(B.BitnetError, match="scratch limit"):
        B.bitnet_quant_weights_noalloc(torch.empty((N, K), dtype=torch.float32, device="meta"))


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_twice():
    dev = torch.device("cuda", 0)
    shapes = [(6912, 2560), (640, 2576)]   # the second call reuses fewer, differently sized blocks
    for call, (N, K) in enumerate(shapes):
        W = synthetic.latent_weights(N, K, seed=900 + call).to(dev)
        Wq_ref, g_ref = B.bitnet_quant_weights(W)
        Wq, g = B.bitnet_quant_weights_noalloc(W)
        torch.cuda.synchronize()
        assert torch.equal(g.view(torch.int32).cpu(), g_ref.view(torch.int32).cpu()), f"call {call}: gamma"
        assert torch.equal(Wq.cpu(), Wq_ref.cpu()), f"call {call}: W_q"
