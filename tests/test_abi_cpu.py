"""The C-ABI library loads and exports every symbol include/bitnet.h declares;
argument validation runs on the host before any device work.  CPU only: no
call here reaches a kernel."""
import ctypes
import os
import re

import pytest

from conftest import ROOT

import bitlinear_bitnet_linear_b200 as bn
from bitlinear_bitnet_linear_b200 import _binding, build

HEADER = os.path.join(ROOT, "include", "bitnet.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return _binding.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(bitnet_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_expected_api():
    names = declared_functions()
    for n in ("bitnet_quant_weights", "bitnet_pack", "bitnet_quant_act", "bitnet_linear"):
        assert n in names
    assert sorted(_binding.EXPORTS) == names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_status_strings(L):
    for s in range(10):
        assert L.bitnet_status_str(s)


def test_workspace_sizes(L):
    assert L.bitnet_workspace_bytes(1, 2560, 2560) >= 256
    big = L.bitnet_workspace_bytes(4096, 2560, 6912)
    assert big >= 256 + 4096 * 2560 + 2 * 4096 * 4
    assert L.bitnet_quant_weights_workspace_bytes(2560, 2560) >= 256 + 16 * 8


FAKE = ctypes.c_void_p(0x10000)          # aligned, never dereferenced: validation fails first
MISALIGNED = ctypes.c_void_p(0x10008)


def test_null_and_shape_errors(L):
    z = ctypes.c_size_t(1 << 20)
    # null weights
    assert L.bitnet_pack(None, 4, 16, FAKE, None, None) == 1
    # K not a multiple of 16, N < 1
    assert L.bitnet_pack(FAKE, 4, 24, FAKE, None, None) == 2
    assert L.bitnet_pack(FAKE, 0, 16, FAKE, None, None) == 2
    # misaligned
    assert L.bitnet_pack(MISALIGNED, 4, 16, FAKE, None, None) == 3
    # dtype
    assert L.bitnet_quant_act(FAKE, 7, 1, 16, None, 1e-5, FAKE, FAKE, None, None) == 4
    # linear: y NULL
    assert L.bitnet_linear(FAKE, 1, 1, 16, FAKE, 4, FAKE, None, 1e-5, None, 1, FAKE, z, None) == 1
    # workspace misaligned
    assert L.bitnet_linear(FAKE, 1, 1, 16, FAKE, 4, FAKE, None, 1e-5, FAKE, 1,
                           ctypes.c_void_p(0x10010), z, None) == 8
    # unknown path
    assert L.bitnet_linear_ex(FAKE, 1, 1, 16, FAKE, 4, FAKE, None, 1e-5, FAKE, 1, FAKE, z, 9, None) == 5
    # wait limit must be positive
    assert L.bitnet_set_wait_limit_us(0) == 2


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="host without a device only")
def test_no_cpu_fallback(L):
    """With valid arguments but no CUDA device the library refuses to run
    (ERR_UNSUPPORTED) instead of computing on the host."""
    z = ctypes.c_size_t(1 << 20)
    assert L.bitnet_linear(FAKE, 1, 1, 16, FAKE, 4, FAKE, None, 1e-5, FAKE, 1, FAKE, z, None) == 5
    assert L.bitnet_pack(FAKE, 4, 16, FAKE, None, None) == 5


def test_binding_refuses_cpu_tensors():
    import torch
    with pytest.raises(ValueError):
        bn.bitnet_pack(torch.zeros((4, 16), dtype=torch.int8))


def _empty_calls(L):
    """Each compute entry point with the dimensions it takes: (call, dims)."""
    F = FAKE
    z = ctypes.c_size_t(1 << 20)
    e = 1e-5
    return {
        "quant_weights": (lambda M, K, N: L.bitnet_quant_weights(F, N, K, 1e-8, F, F, F, z, None), "KN"),
        "ternarise": (lambda M, K, N: L.bitnet_ternarise(F, N, K, F, 1e-8, F, None), "KN"),
        "pack": (lambda M, K, N: L.bitnet_pack(F, N, K, F, None, None), "KN"),
        "unpack": (lambda M, K, N: L.bitnet_unpack(F, N, K, F, None, None), "KN"),
        "quant_act": (lambda M, K, N: L.bitnet_quant_act(F, 1, M, K, None, e, F, F, None, None), "MK"),
        "quant_act_relu2": (lambda M, K, N: L.bitnet_quant_act_relu2(F, F, 1, M, K, None, e, F, F, None, None),
                            "MK"),
        "linear": (lambda M, K, N: L.bitnet_linear(F, 1, M, K, F, N, F, None, e, F, 1, F, z, None), "MKN"),
        "linear_ex": (lambda M, K, N: L.bitnet_linear_ex(F, 1, M, K, F, N, F, None, e, F, 1, F, z, 2, None), "MKN"),
        "linear_q": (lambda M, K, N: L.bitnet_linear_q(F, F, None, M, K, F, N, F, F, 1, None, F, z, 0, None), "MKN"),
        "linear_relu2": (lambda M, K, N: L.bitnet_linear_relu2(F, F, 1, M, K, F, N, F, None, e, None, F, 1, F, z,
                                                               None), "MKN"),
        "quant_weights_b1": (lambda M, K, N: L.bitnet_quant_weights_b1(F, N, K, F, F, F, z, None), "KN"),
        "pack_b1": (lambda M, K, N: L.bitnet_pack_b1(F, N, K, F, None, None), "KN"),
        "unpack_b1": (lambda M, K, N: L.bitnet_unpack_b1(F, N, K, F, None), "KN"),
        "linear_b1": (lambda M, K, N: L.bitnet_linear_b1(F, 1, M, K, F, N, F, None, e, F, 1, F, z, None), "MKN"),
        "pack_t3": (lambda M, K, N: L.bitnet_pack_t3(F, N, K, F, None, None), "KN"),
        "unpack_t3": (lambda M, K, N: L.bitnet_unpack_t3(F, N, K, F, None, None), "KN"),
        "linear_t3": (lambda M, K, N: L.bitnet_linear_t3(F, 1, K, F, N, F, None, e, F, 1, F, z, None), "KN"),
        "quant_weights_noalloc": (lambda M, K, N: L.bitnet_quant_weights_noalloc(F, N, K, 1e-8, F, F, None), "KN"),
    }


def test_empty_and_negative_dimensions_rejected(L):
    """Empty inputs: every compute entry point answers BITNET_ERR_SHAPE for
    a zero or negative M, K or N it takes, before any device work."""
    base = {"M": 1, "K": 128, "N": 8}
    for name, (call, dims) in _empty_calls(L).items():
        for d in dims:
            for bad in (0, -16):
                args = dict(base)
                args[d] = bad
                assert call(args["M"], args["K"], args["N"]) == 2, (name, d, bad)


def test_empty_grouped_call_rejected(L):
    """A grouped call with no problems (or more than 256) is a shape error;
    the problem table is not read."""
    z = ctypes.c_size_t(1 << 20)
    for count in (0, -1, 257):
        assert L.bitnet_linear_grouped(FAKE, count, 1, 1, 1e-5, 1, FAKE, z, None) == 2
        assert L.bitnet_linear_grouped_b1(FAKE, count, 1, 1e-5, 1, FAKE, z, None) == 2
        assert L.bitnet_linear_grouped_t3(FAKE, count, 1, 1e-5, 1, FAKE, z, None) == 2
