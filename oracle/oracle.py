"""CPU oracle for the BitLinear path -- TEST INFRASTRUCTURE ONLY.

Thin ctypes wrapper over ``bitnet_oracle.c`` (plain scalar C).  Only the
tests, the smoke check and the benchmark's CPU-baseline leg may import this
module; the product library never does, and this module imports nothing from
the product package.

Each function cites the page passage its C counterpart restates (see the C
file's header for the page names).  Inputs and outputs are numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
# BITNET_ORACLE_SRC / BITNET_ORACLE_LIB point the module at another copy of
# the C source and its build: the mutation tests plant a mistake in a copy
# and check that the pins reject it.
_SRC = os.environ.get("BITNET_ORACLE_SRC") or os.path.join(_HERE, "bitnet_oracle.c")
_LIB_PATH = os.environ.get("BITNET_ORACLE_LIB") or os.path.join(_HERE, "liboracle.so")

# The activation floor that guards an all-zero row (the pages are silent).
FLOOR_EPS = 1e-5
# [Gartu] round(w / (beta + 1e-8)).
W_EPS = 1e-8


def build(force: bool = False) -> str:
    """Compile the oracle with IEEE semantics (no fast-math, no contraction)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
           "-ffp-contract=off", "-fexcess-precision=standard",
           "-o", _LIB_PATH + ".tmp", _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(_LIB_PATH + ".tmp", _LIB_PATH)
    return _LIB_PATH


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        P, I64, F, D = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_double
        L.orc_abs_sum.argtypes = [P, I64]; L.orc_abs_sum.restype = D
        L.orc_gamma.argtypes = [P, I64]; L.orc_gamma.restype = F
        L.orc_ternarise.argtypes = [P, I64, F, F, P]; L.orc_ternarise.restype = None
        L.orc_pack.argtypes = [P, I64, I64, P]; L.orc_pack.restype = I64
        L.orc_unpack.argtypes = [P, I64, I64, P]; L.orc_unpack.restype = I64
        L.orc_quant_act.argtypes = [P, I64, I64, P, F, F, P, P, P]
        L.orc_quant_act.restype = None
        L.orc_linear_i32.argtypes = [P, I64, I64, P, I64, P]; L.orc_linear_i32.restype = None
        L.orc_output.argtypes = [P, I64, I64, F, P, P]; L.orc_output.restype = None
        L.orc_to_bf16.argtypes = [P, I64, P]; L.orc_to_bf16.restype = None
        L.orc_relu2_gate.argtypes = [P, P, I64, P]; L.orc_relu2_gate.restype = None
        L.orc_binarise.argtypes = [P, I64, P]; L.orc_binarise.restype = None
        L.orc_pack_b1.argtypes = [P, I64, I64, P]; L.orc_pack_b1.restype = I64
        L.orc_unpack_b1.argtypes = [P, I64, I64, P]; L.orc_unpack_b1.restype = None
        L.orc_t3_row_bytes.argtypes = [I64]; L.orc_t3_row_bytes.restype = I64
        L.orc_pack_t3.argtypes = [P, I64, I64, P]; L.orc_pack_t3.restype = I64
        L.orc_unpack_t3.argtypes = [P, I64, I64, P]; L.orc_unpack_t3.restype = I64
        L.orc_output_resid.argtypes = [P, I64, I64, F, P, P, P]; L.orc_output_resid.restype = None
        _lib = L
    return _lib


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def abs_sum(W: np.ndarray) -> float:
    """Correctly rounded binary64 value of sum |W| ([Gartu] w.abs().mean() numerator)."""
    W = _c(W, np.float32)
    return float(lib().orc_abs_sum(_p(W), W.size))


def gamma(W: np.ndarray) -> np.float32:
    """Absmean scale gamma = mean |W| ([KeyTech] absmean; [Gartu] beta)."""
    W = _c(W, np.float32)
    return np.float32(lib().orc_gamma(_p(W), W.size))


def ternarise(W: np.ndarray, g: float, eps: float = W_EPS) -> np.ndarray:
    """W_q = clamp(round(W / (gamma + eps)), -1, 1) ([Gartu] BitLinear.forward)."""
    W = _c(W, np.float32)
    out = np.empty(W.shape, np.int8)
    lib().orc_ternarise(_p(W), W.size, float(np.float32(g)), float(np.float32(eps)), _p(out))
    return out


def quant_weights(W: np.ndarray, eps: float = W_EPS):
    """(W_q, gamma): the absmean ternary weight quantiser ([KeyTech], [Gartu])."""
    g = gamma(W)
    return ternarise(W, g, eps), g


def pack(Wq: np.ndarray):
    """2 bits per weight ([Notes] bit-packing).  Returns (packed [N, K/4] uint8, n_invalid)."""
    Wq = _c(Wq, np.int8)
    N, K = Wq.shape
    out = np.empty((N, K // 4), np.uint8)
    bad = lib().orc_pack(_p(Wq), N, K, _p(out))
    return out, int(bad)


def unpack(Wp: np.ndarray, K: int):
    """Inverse of ``pack``.  Returns (W_q [N, K] int8, n_code3)."""
    Wp = _c(Wp, np.uint8)
    N = Wp.shape[0]
    out = np.empty((N, K), np.int8)
    bad = lib().orc_unpack(_p(Wp), N, K, _p(out))
    return out, int(bad)


def quant_act(x: np.ndarray, gain: np.ndarray | None = None, rms_eps: float = 1e-5,
              floor_eps: float = FLOOR_EPS):
    """Per-token absmax int8 ([KeyTech]; [HN-b158] int8 activations), optional
    fused RMSNorm gain.  Returns (x_q int8 [M,K], scale f32 [M], xsum int32 [M])."""
    x = _c(x, np.float32)
    M, K = x.shape
    xq = np.empty((M, K), np.int8)
    sc = np.empty(M, np.float32)
    xs = np.empty(M, np.int32)
    gp = None
    if gain is not None:
        gain = _c(gain, np.float32)
        gp = _p(gain)
    lib().orc_quant_act(_p(x), M, K, gp, float(np.float32(rms_eps)),
                        float(np.float32(floor_eps)), _p(xq), _p(sc), _p(xs))
    return xq, sc, xs


def linear_i32(xq: np.ndarray, Wq: np.ndarray) -> np.ndarray:
    """acc = x_q @ W_q^T in exact integers ([Gartu] F.linear)."""
    xq = _c(xq, np.int8)
    Wq = _c(Wq, np.int8)
    M, K = xq.shape
    N = Wq.shape[0]
    acc = np.empty((M, N), np.int32)
    lib().orc_linear_i32(_p(xq), M, K, _p(Wq), N, _p(acc))
    return acc


def output(acc: np.ndarray, g: float, scale: np.ndarray) -> np.ndarray:
    """y = acc * (gamma * s_m) in binary32."""
    acc = _c(acc, np.int32)
    scale = _c(scale, np.float32)
    M, N = acc.shape
    y = np.empty((M, N), np.float32)
    lib().orc_output(_p(acc), M, N, float(np.float32(g)), _p(scale), _p(y))
    return y


def binarise(W: np.ndarray) -> np.ndarray:
    """BitNet b1 weights: +1 where W >= 0, else -1 ([Gartu] binary BitLinear)."""
    W = _c(W, np.float32)
    out = np.empty(W.shape, np.int8)
    lib().orc_binarise(_p(W), W.size, _p(out))
    return out


def quant_weights_b1(W: np.ndarray):
    """(W_b, beta): signs and the absmean scale."""
    return binarise(W), gamma(W)


def pack_b1(Wb: np.ndarray):
    """1 bit per weight.  Returns (packed [N, K/8] uint8, n_invalid)."""
    Wb = _c(Wb, np.int8)
    N, K = Wb.shape
    out = np.empty((N, K // 8), np.uint8)
    bad = lib().orc_pack_b1(_p(Wb), N, K, _p(out))
    return out, int(bad)


def unpack_b1(Wp: np.ndarray, K: int) -> np.ndarray:
    Wp = _c(Wp, np.uint8)
    N = Wp.shape[0]
    out = np.empty((N, K), np.int8)
    lib().orc_unpack_b1(_p(Wp), N, K, _p(out))
    return out


def t3_row_bytes(K: int) -> int:
    return int(lib().orc_t3_row_bytes(K))


def pack_t3(Wq: np.ndarray):
    """Base-3, five weights per byte.  Returns (packed [N, t3_row_bytes(K)] uint8, n_invalid)."""
    Wq = _c(Wq, np.int8)
    N, K = Wq.shape
    out = np.empty((N, t3_row_bytes(K)), np.uint8)
    bad = lib().orc_pack_t3(_p(Wq), N, K, _p(out))
    return out, int(bad)


def unpack_t3(Wp: np.ndarray, K: int):
    Wp = _c(Wp, np.uint8)
    N = Wp.shape[0]
    out = np.empty((N, K), np.int8)
    bad = lib().orc_unpack_t3(_p(Wp), N, K, _p(out))
    return out, int(bad)


def relu2_gate(gate: np.ndarray, up: np.ndarray) -> np.ndarray:
    """t = max(gate, 0)^2 * up in binary32, (r * r) * u."""
    gate = _c(gate, np.float32)
    up = _c(up, np.float32)
    assert gate.shape == up.shape
    t = np.empty(gate.shape, np.float32)
    lib().orc_relu2_gate(_p(gate), _p(up), gate.size, _p(t))
    return t


def output_resid(acc: np.ndarray, g: float, scale: np.ndarray, resid: np.ndarray) -> np.ndarray:
    """y = resid + acc * (gamma * s_m) in binary32."""
    acc = _c(acc, np.int32)
    scale = _c(scale, np.float32)
    resid = _c(resid, np.float32)
    M, N = acc.shape
    assert resid.shape == (M, N)
    y = np.empty((M, N), np.float32)
    lib().orc_output_resid(_p(acc), M, N, float(np.float32(g)), _p(scale), _p(resid), _p(y))
    return y


def to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """binary32 -> bfloat16 bit patterns (uint16), round to nearest even."""
    v = _c(v, np.float32)
    out = np.empty(v.shape, np.uint16)
    lib().orc_to_bf16(_p(v), v.size, _p(out))
    return out


def bitlinear(x: np.ndarray, Wq: np.ndarray, g: float, gain: np.ndarray | None = None,
              rms_eps: float = 1e-5):
    """Whole forward: returns (y f32, x_q, scale, xsum, acc)."""
    xq, sc, xs = quant_act(x, gain, rms_eps)
    acc = linear_i32(xq, Wq)
    return output(acc, g, sc), xq, sc, xs, acc
