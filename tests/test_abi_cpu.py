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
