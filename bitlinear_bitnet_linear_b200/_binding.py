"""ctypes binding for libbitnet.so: argument marshalling only.

Every function here has the name of the C entry point it calls
(include/bitnet.h), takes torch CUDA tensors, passes their device pointers
and the current CUDA stream, and raises BitnetError on a non-OK status.
No arithmetic of the method happens in Python; there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbitnet.so")

OK = 0
STATUS_NAMES = {0: "OK", 1: "ERR_NULL", 2: "ERR_SHAPE", 3: "ERR_ALIGN", 4: "ERR_DTYPE",
                5: "ERR_UNSUPPORTED", 6: "ERR_CUDA", 7: "ERR_TIMEOUT", 8: "ERR_WORKSPACE",
                9: "ERR_VALUE"}
F32, BF16 = 0, 1
PATH_AUTO, PATH_GEMV, PATH_TC = 0, 1, 2

# every symbol declared in include/bitnet.h
EXPORTS = ("bitnet_workspace_bytes", "bitnet_quant_weights_workspace_bytes", "bitnet_workspace_init",
           "bitnet_get_error", "bitnet_status_str", "bitnet_quant_weights", "bitnet_ternarise",
           "bitnet_pack", "bitnet_unpack", "bitnet_quant_act", "bitnet_linear", "bitnet_linear_ex",
           "bitnet_linear_q", "bitnet_linear_grouped", "bitnet_linear_relu2", "bitnet_quant_act_relu2",
           "bitnet_quant_weights_b1", "bitnet_pack_b1", "bitnet_unpack_b1", "bitnet_linear_b1",
           "bitnet_linear_grouped_b1", "bitnet_t3_row_bytes", "bitnet_pack_t3", "bitnet_unpack_t3",
           "bitnet_linear_t3", "bitnet_linear_grouped_t3",
           "bitnet_quant_weights_noalloc",
           "bitnet_set_wait_limit_us", "bitnet_watchdog_selftest", "bitnet_debug_stream_plan")


class GemvProblem(ctypes.Structure):
    """Mirror of bitnet_gemv_problem (include/bitnet.h)."""
    _fields_ = [("x", ctypes.c_void_p), ("Wp", ctypes.c_void_p), ("gamma", ctypes.c_void_p),
                ("rms_gain", ctypes.c_void_p), ("y", ctypes.c_void_p), ("K", ctypes.c_int64),
                ("N", ctypes.c_int64)]


class BitnetError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)} ({status_str(status)})")


_lib = None


def lib() -> ctypes.CDLL:
    """Load libbitnet.so (built in-tree by build.py); raise if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libbitnet.so not built ({LIB_PATH}); run bitlinear_bitnet_linear_b200.build.build()")
    L = ctypes.CDLL(LIB_PATH)
    P, I64, I32, U32, F, SZ = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_uint32,
                               ctypes.c_float, ctypes.c_size_t)
    sig = {
        "bitnet_workspace_bytes": ([I64, I64, I64], SZ),
        "bitnet_quant_weights_workspace_bytes": ([I64, I64], SZ),
        "bitnet_workspace_init": ([P, SZ, P], I32),
        "bitnet_get_error": ([P, P], I32),
        "bitnet_status_str": ([I32], ctypes.c_char_p),
        "bitnet_quant_weights": ([P, I64, I64, F, P, P, P, SZ, P], I32),
        "bitnet_ternarise": ([P, I64, I64, P, F, P, P], I32),
        "bitnet_quant_weights_noalloc": ([P, I64, I64, F, P, P, P], I32),
        "bitnet_pack": ([P, I64, I64, P, P, P], I32),
        "bitnet_unpack": ([P, I64, I64, P, P, P], I32),
        "bitnet_quant_act": ([P, I32, I64, I64, P, F, P, P, P, P], I32),
        "bitnet_quant_act_relu2": ([P, P, I32, I64, I64, P, F, P, P, P, P], I32),
        "bitnet_quant_weights_b1": ([P, I64, I64, P, P, P, SZ, P], I32),
        "bitnet_pack_b1": ([P, I64, I64, P, P, P], I32),
        "bitnet_unpack_b1": ([P, I64, I64, P, P], I32),
        "bitnet_linear_b1": ([P, I32, I64, I64, P, I64, P, P, F, P, I32, P, SZ, P], I32),
        "bitnet_linear_grouped_b1": ([P, I32, I32, F, I32, P, SZ, P], I32),
        "bitnet_t3_row_bytes": ([I64], I64),
        "bitnet_pack_t3": ([P, I64, I64, P, P, P], I32),
        "bitnet_unpack_t3": ([P, I64, I64, P, P, P], I32),
        "bitnet_linear_t3": ([P, I32, I64, P, I64, P, P, F, P, I32, P, SZ, P], I32),
        "bitnet_linear_grouped_t3": ([P, I32, I32, F, I32, P, SZ, P], I32),
        "bitnet_linear_relu2": ([P, P, I32, I64, I64, P, I64, P, P, F, P, P, I32, P, SZ, P], I32),
        "bitnet_linear": ([P, I32, I64, I64, P, I64, P, P, F, P, I32, P, SZ, P], I32),
        "bitnet_linear_ex": ([P, I32, I64, I64, P, I64, P, P, F, P, I32, P, SZ, I32, P], I32),
        "bitnet_linear_q": ([P, P, P, I64, I64, P, I64, P, P, I32, P, P, SZ, I32, P], I32),
        "bitnet_linear_grouped": ([P, I32, I64, I32, F, I32, P, SZ, P], I32),
        "bitnet_set_wait_limit_us": ([U32], I32),
        "bitnet_watchdog_selftest": ([P, SZ, U32, P], I32),
        "bitnet_debug_stream_plan": ([P, P, I32, I64, I32, I32, I32, I32, P, P, P], I32),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    _lib = L
    return L


def status_str(s: int) -> str:
    try:
        return lib().bitnet_status_str(int(s)).decode()
    except Exception:  # pragma: no cover - only when the library is absent
        return "?"


def _check(st: int, what: str) -> None:
    if st != OK:
        raise BitnetError(st, what)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must be on a CUDA device")
    if t.device.index != torch.cuda.current_device():
        # the library launches on the current device
        raise ValueError(f"tensor is on {t.device}; the current device is cuda:{torch.cuda.current_device()}")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _xdtype(t) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise ValueError(f"unsupported dtype {t.dtype}")


def _ydtype(d) -> int:
    return {torch.float32: F32, torch.bfloat16: BF16}[d]


# --------------------------------------------------------------------------
# workspace
# --------------------------------------------------------------------------

def bitnet_workspace_bytes(M: int, K: int, N: int) -> int:
    return int(lib().bitnet_workspace_bytes(M, K, N))


def bitnet_quant_weights_workspace_bytes(N: int, K: int) -> int:
    return int(lib().bitnet_quant_weights_workspace_bytes(N, K))


def new_workspace(nbytes: int, device=None) -> torch.Tensor:
    """A zeroed device buffer usable as a workspace (torch blocks are 512-byte aligned)."""
    n = max(256, (int(nbytes) + 255) // 256 * 256)
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def bitnet_workspace_init(ws: torch.Tensor, stream=None) -> None:
    _check(lib().bitnet_workspace_init(_ptr(ws), ws.numel(), _stream(stream)), "bitnet_workspace_init")


def bitnet_get_error(ws: torch.Tensor, stream=None) -> int:
    """Synchronise and return (and clear) the workspace's device status."""
    return int(lib().bitnet_get_error(_ptr(ws), _stream(stream)))


def bitnet_set_wait_limit_us(limit_us: int) -> None:
    _check(lib().bitnet_set_wait_limit_us(int(limit_us)), "bitnet_set_wait_limit_us")


def bitnet_watchdog_selftest(ws: torch.Tensor, limit_us: int, stream=None) -> None:
    _check(lib().bitnet_watchdog_selftest(_ptr(ws), ws.numel(), int(limit_us), _stream(stream)),
           "bitnet_watchdog_selftest")


def bitnet_debug_stream_plan(shapes, M: int, bits: int = 2, prequant: bool = False, sms: int = 148,
                             smem_optin: int = 232448) -> dict:
    """The streaming GEMV's plan for problems [(K, N), ...] on a described
    device (host computation only; no GPU needed)."""
    n = len(shapes)
    Ks = (ctypes.c_int64 * n)(*[int(k) for k, _ in shapes])
    Ns = (ctypes.c_int64 * n)(*[int(v) for _, v in shapes])
    shape = (ctypes.c_int64 * 5)()
    rows = (ctypes.c_int32 * n)()
    task = (ctypes.c_int32 * n)()
    _check(lib().bitnet_debug_stream_plan(Ks, Ns, n, int(M), int(bits), int(bool(prequant)), int(sms),
                                          int(smem_optin), shape, rows, task), "bitnet_debug_stream_plan")
    return {"grid": shape[0], "smem": shape[1], "nxb": shape[2], "nslots": shape[3], "slot_bytes": shape[4],
            "rows": list(rows), "task": list(task)}


# --------------------------------------------------------------------------
# weight preparation
# --------------------------------------------------------------------------

def bitnet_quant_weights(W: torch.Tensor, eps: float = 1e-8, Wq: torch.Tensor | None = None,
                         gamma: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                         want_wq: bool = True, stream=None):
    """Returns (Wq int8 [N, K] or None, gamma float32 [1]) on W's device."""
    N, K = W.shape
    if want_wq and Wq is None:
        Wq = torch.empty((N, K), dtype=torch.int8, device=W.device)
    if gamma is None:
        gamma = torch.empty(1, dtype=torch.float32, device=W.device)
    if ws is None:
        ws = new_workspace(bitnet_quant_weights_workspace_bytes(N, K), W.device)
    _check(lib().bitnet_quant_weights(_ptr(W), N, K, float(eps), _ptr(Wq) if want_wq else None, _ptr(gamma),
                                      _ptr(ws), ws.numel(), _stream(stream)), "bitnet_quant_weights")
    return Wq, gamma


# Largest N*K bitnet_quant_weights_noalloc accepts: 2048 blocks of 2^24 weights.
NOALLOC_MAX_ELEMENTS = 2048 * (1 << 24)


def bitnet_quant_weights_noalloc(W: torch.Tensor, eps: float = 1e-8, Wq: torch.Tensor | None = None,
                                 gamma: torch.Tensor | None = None, want_wq: bool = True, stream=None):
    """bitnet_quant_weights without a workspace (the library's own scratch).
    Outputs are allocated here only when not given."""
    N, K = W.shape
    if N * K > NOALLOC_MAX_ELEMENTS:
        raise BitnetError(2, f"bitnet_quant_weights_noalloc: N*K = {N * K} exceeds the scratch limit "
                             f"{NOALLOC_MAX_ELEMENTS} (use bitnet_quant_weights with a workspace)")
    if want_wq and Wq is None:
        Wq = torch.empty((N, K), dtype=torch.int8, device=W.device)
    if gamma is None:
        gamma = torch.empty(1, dtype=torch.float32, device=W.device)
    _check(lib().bitnet_quant_weights_noalloc(_ptr(W), N, K, float(eps), _ptr(Wq) if want_wq else None,
                                              _ptr(gamma), _stream(stream)), "bitnet_quant_weights_noalloc")
    return Wq, gamma


def bitnet_ternarise(W: torch.Tensor, gamma: torch.Tensor, eps: float = 1e-8, Wq=None, stream=None):
    N, K = W.shape
    if Wq is None:
        Wq = torch.empty((N, K), dtype=torch.int8, device=W.device)
    _check(lib().bitnet_ternarise(_ptr(W), N, K, _ptr(gamma), float(eps), _ptr(Wq), _stream(stream)),
           "bitnet_ternarise")
    return Wq


def bitnet_pack(Wq: torch.Tensor, Wp=None, n_invalid=None, stream=None):
    N, K = Wq.shape
    if Wp is None:
        Wp = torch.empty((N, K // 4), dtype=torch.uint8, device=Wq.device)
    _check(lib().bitnet_pack(_ptr(Wq), N, K, _ptr(Wp), _ptr(n_invalid), _stream(stream)), "bitnet_pack")
    return Wp


def bitnet_unpack(Wp: torch.Tensor, K: int, Wq=None, n_invalid=None, stream=None):
    N = Wp.shape[0]
    if Wq is None:
        Wq = torch.empty((N, K), dtype=torch.int8, device=Wp.device)
    _check(lib().bitnet_unpack(_ptr(Wp), N, K, _ptr(Wq), _ptr(n_invalid), _stream(stream)), "bitnet_unpack")
    return Wq


# --------------------------------------------------------------------------
# per-call path
# --------------------------------------------------------------------------

def bitnet_quant_act(x: torch.Tensor, rms_gain: torch.Tensor | None = None, rms_eps: float = 1e-5,
                     xq=None, x_scale=None, x_sum=None, want_sum: bool = True, stream=None):
    M, K = x.shape
    if xq is None:
        xq = torch.empty((M, K), dtype=torch.int8, device=x.device)
    if x_scale is None:
        x_scale = torch.empty(M, dtype=torch.float32, device=x.device)
    if want_sum and x_sum is None:
        x_sum = torch.empty(M, dtype=torch.int32, device=x.device)
    _check(lib().bitnet_quant_act(_ptr(x), _xdtype(x), M, K, _ptr(rms_gain), float(rms_eps), _ptr(xq),
                                  _ptr(x_scale), _ptr(x_sum) if want_sum else None, _stream(stream)),
           "bitnet_quant_act")
    return xq, x_scale, (x_sum if want_sum else None)


def bitnet_linear(x: torch.Tensor, Wp: torch.Tensor, gamma: torch.Tensor, N: int | None = None,
                  rms_gain: torch.Tensor | None = None, rms_eps: float = 1e-5, y=None,
                  y_dtype=torch.bfloat16, ws=None, path: int = PATH_AUTO, stream=None):
    M, K = x.shape
    N = Wp.shape[0] if N is None else N
    if y is None:
        y = torch.empty((M, N), dtype=y_dtype, device=x.device)
    if ws is None:
        ws = new_workspace(bitnet_workspace_bytes(M, K, N), x.device)
    _check(lib().bitnet_linear_ex(_ptr(x), _xdtype(x), M, K, _ptr(Wp), N, _ptr(gamma), _ptr(rms_gain),
                                  float(rms_eps), _ptr(y), _ydtype(y.dtype), _ptr(ws), ws.numel(), int(path),
                                  _stream(stream)), "bitnet_linear")
    return y


def bitnet_quant_weights_b1(W: torch.Tensor, Wb: torch.Tensor | None = None, beta: torch.Tensor | None = None,
                            ws: torch.Tensor | None = None, want_wb: bool = True, stream=None):
    """BitNet b1: (W_b int8 +-1 [N, K] or None, beta float32 [1])."""
    N, K = W.shape
    if want_wb and Wb is None:
        Wb = torch.empty((N, K), dtype=torch.int8, device=W.device)
    if beta is None:
        beta = torch.empty(1, dtype=torch.float32, device=W.device)
    if ws is None:
        ws = new_workspace(bitnet_quant_weights_workspace_bytes(N, K), W.device)
    _check(lib().bitnet_quant_weights_b1(_ptr(W), N, K, _ptr(Wb) if want_wb else None, _ptr(beta), _ptr(ws),
                                         ws.numel(), _stream(stream)), "bitnet_quant_weights_b1")
    return (Wb if want_wb else None), beta


def bitnet_pack_b1(Wb: torch.Tensor, n_invalid: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    N, K = Wb.shape
    Wp = torch.empty((N, K // 8), dtype=torch.uint8, device=Wb.device)
    _check(lib().bitnet_pack_b1(_ptr(Wb), N, K, _ptr(Wp), _ptr(n_invalid), _stream(stream)), "bitnet_pack_b1")
    return Wp


def bitnet_unpack_b1(Wp: torch.Tensor, K: int, stream=None) -> torch.Tensor:
    N = Wp.shape[0]
    Wb = torch.empty((N, K), dtype=torch.int8, device=Wp.device)
    _check(lib().bitnet_unpack_b1(_ptr(Wp), N, K, _ptr(Wb), _stream(stream)), "bitnet_unpack_b1")
    return Wb


def bitnet_linear_b1(x: torch.Tensor, Wp: torch.Tensor, beta: torch.Tensor, N: int | None = None,
                     rms_gain: torch.Tensor | None = None, rms_eps: float = 1e-5, y=None,
                     y_dtype=torch.bfloat16, ws=None, stream=None):
    M, K = x.shape
    N = Wp.shape[0] if N is None else N
    if y is None:
        y = torch.empty((M, N), dtype=y_dtype, device=x.device)
    if ws is None:
        ws = new_workspace(bitnet_workspace_bytes(M, K, N), x.device)
    _check(lib().bitnet_linear_b1(_ptr(x), _xdtype(x), M, K, _ptr(Wp), N, _ptr(beta), _ptr(rms_gain),
                                  float(rms_eps), _ptr(y), _ydtype(y.dtype), _ptr(ws), ws.numel(),
                                  _stream(stream)), "bitnet_linear_b1")
    return y


def bitnet_t3_row_bytes(K: int) -> int:
    return int(lib().bitnet_t3_row_bytes(K))


def bitnet_pack_t3(Wq: torch.Tensor, n_invalid: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Base-3: five ternary weights per byte, [N, bitnet_t3_row_bytes(K)] uint8."""
    N, K = Wq.shape
    Wp = torch.empty((N, bitnet_t3_row_bytes(K)), dtype=torch.uint8, device=Wq.device)
    _check(lib().bitnet_pack_t3(_ptr(Wq), N, K, _ptr(Wp), _ptr(n_invalid), _stream(stream)), "bitnet_pack_t3")
    return Wp


def bitnet_unpack_t3(Wp: torch.Tensor, K: int, n_invalid: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    N = Wp.shape[0]
    Wq = torch.empty((N, K), dtype=torch.int8, device=Wp.device)
    _check(lib().bitnet_unpack_t3(_ptr(Wp), N, K, _ptr(Wq), _ptr(n_invalid), _stream(stream)), "bitnet_unpack_t3")
    return Wq


def bitnet_linear_t3(x: torch.Tensor, Wp: torch.Tensor, gamma: torch.Tensor, N: int | None = None,
                     rms_gain: torch.Tensor | None = None, rms_eps: float = 1e-5, y=None,
                     y_dtype=torch.bfloat16, ws=None, stream=None):
    """One token through base-3 packed weights."""
    M, K = x.shape
    if M != 1:
        raise ValueError("bitnet_linear_t3 takes one token")
    N = Wp.shape[0] if N is None else N
    if y is None:
        y = torch.empty((1, N), dtype=y_dtype, device=x.device)
    if ws is None:
        ws = new_workspace(bitnet_workspace_bytes(1, K, N), x.device)
    _check(lib().bitnet_linear_t3(_ptr(x), _xdtype(x), K, _ptr(Wp), N, _ptr(gamma), _ptr(rms_gain),
                                  float(rms_eps), _ptr(y), _ydtype(y.dtype), _ptr(ws), ws.numel(),
                                  _stream(stream)), "bitnet_linear_t3")
    return y


def bitnet_quant_act_relu2(gate: torch.Tensor, up: torch.Tensor, rms_gain: torch.Tensor | None = None,
                           rms_eps: float = 1e-5, xq=None, x_scale=None, x_sum=None, stream=None):
    """Codes, scales and code sums of t = max(gate, 0)^2 * up."""
    M, K = gate.shape
    if up.shape != gate.shape or up.dtype != gate.dtype:
        raise ValueError("gate and up must have the same shape and dtype")
    if xq is None:
        xq = torch.empty((M, K), dtype=torch.int8, device=gate.device)
    if x_scale is None:
        x_scale = torch.empty(M, dtype=torch.float32, device=gate.device)
    if x_sum is None:
        x_sum = torch.empty(M, dtype=torch.int32, device=gate.device)
    _check(lib().bitnet_quant_act_relu2(_ptr(gate), _ptr(up), _xdtype(gate), M, K, _ptr(rms_gain), float(rms_eps),
                                        _ptr(xq), _ptr(x_scale), _ptr(x_sum), _stream(stream)),
           "bitnet_quant_act_relu2")
    return xq, x_scale, x_sum


def bitnet_linear_relu2(gate: torch.Tensor, up: torch.Tensor, Wp: torch.Tensor, gamma: torch.Tensor,
                        N: int | None = None, rms_gain: torch.Tensor | None = None, rms_eps: float = 1e-5,
                        resid: torch.Tensor | None = None, y=None, y_dtype=torch.bfloat16, ws=None, stream=None):
    """Down projection of the ReLU^2-gated input, plus an optional residual."""
    M, K = gate.shape
    if up.shape != gate.shape or up.dtype != gate.dtype:
        raise ValueError("gate and up must have the same shape and dtype")
    N = Wp.shape[0] if N is None else N
    if y is None:
        y = torch.empty((M, N), dtype=y_dtype if resid is None else resid.dtype, device=gate.device)
    if resid is not None and (resid.shape != (M, N) or resid.dtype != y.dtype):
        raise ValueError("resid must be [M, N] of y's dtype")
    if ws is None:
        ws = new_workspace(bitnet_workspace_bytes(M, K, N), gate.device)
    _check(lib().bitnet_linear_relu2(_ptr(gate), _ptr(up), _xdtype(gate), M, K, _ptr(Wp), N, _ptr(gamma),
                                     _ptr(rms_gain), float(rms_eps), _ptr(resid), _ptr(y), _ydtype(y.dtype),
                                     _ptr(ws), ws.numel(), _stream(stream)), "bitnet_linear_relu2")
    return y


def bitnet_linear_q(xq: torch.Tensor, x_scale: torch.Tensor, Wp: torch.Tensor, gamma: torch.Tensor,
                    x_sum: torch.Tensor | None = None, y=None, y_dtype=torch.float32, want_y: bool = True,
                    acc=None, want_acc: bool = False, ws=None, path: int = PATH_AUTO, stream=None):
    M, K = xq.shape
    N = Wp.shape[0]
    if want_y and y is None:
        y = torch.empty((M, N), dtype=y_dtype, device=xq.device)
    if want_acc and acc is None:
        acc = torch.empty((M, N), dtype=torch.int32, device=xq.device)
    if ws is None:
        ws = new_workspace(bitnet_workspace_bytes(M, K, N), xq.device)
    _check(lib().bitnet_linear_q(_ptr(xq), _ptr(x_scale), _ptr(x_sum), M, K, _ptr(Wp), N, _ptr(gamma),
                                 _ptr(y) if want_y else None, _ydtype(y.dtype) if want_y else F32,
                                 _ptr(acc) if want_acc else None, _ptr(ws), ws.numel(), int(path),
                                 _stream(stream)), "bitnet_linear_q")
    return y, acc


def bitnet_linear_grouped(problems, rms_eps: float = 1e-5, ws=None, stream=None, _keep=None):
    """problems: sequence of (x, Wp, gamma, rms_gain or None, y) device tensors,
    all with the same M rows and dtypes.  One launch; see include/bitnet.h."""
    arr = (GemvProblem * len(problems))()
    M = problems[0][0].shape[0]
    xd = _xdtype(problems[0][0])
    yd = _ydtype(problems[0][4].dtype)
    for i, (x, Wp, gamma, gain, y) in enumerate(problems):
        if x.shape[0] != M or _xdtype(x) != xd or _ydtype(y.dtype) != yd:
            raise ValueError("all problems need the same M and dtypes")
        arr[i] = GemvProblem(_ptr(x).value, _ptr(Wp).value, _ptr(gamma).value,
                             None if gain is None else _ptr(gain).value, _ptr(y).value,
                             x.shape[1], Wp.shape[0])
    if ws is None:
        ws = new_workspace(256, problems[0][0].device)
    _check(lib().bitnet_linear_grouped(ctypes.cast(arr, ctypes.c_void_p), len(problems), M, xd, float(rms_eps), yd,
                                       _ptr(ws), ws.numel(), _stream(stream)), "bitnet_linear_grouped")


class GroupedCall:
    """A prepared grouped call: the problem table is built once and reused
    (for CUDA-graph capture or repeated launches)."""

    def __init__(self, problems, rms_eps: float = 1e-5, ws=None, bits: int = 2):
        self.arr = (GemvProblem * len(problems))()
        self.M = problems[0][0].shape[0]
        self.xd = _xdtype(problems[0][0])
        self.yd = _ydtype(problems[0][4].dtype)
        self.keep = list(problems)
        for i, (x, Wp, gamma, gain, y) in enumerate(problems):
            self.arr[i] = GemvProblem(_ptr(x).value, _ptr(Wp).value, _ptr(gamma).value,
                                      None if gain is None else _ptr(gain).value, _ptr(y).value,
                                      x.shape[1], Wp.shape[0])
        self.n = len(problems)
        self.bits = int(bits)   # 2: ternary codes (bitnet_pack); 1: BitNet b1 signs (bitnet_pack_b1); 3: base-3
        self.eps = float(rms_eps)
        self.ws = ws if ws is not None else new_workspace(256, problems[0][0].device)

    def __call__(self, stream=None):
        if self.bits == 3:
            _check(lib().bitnet_linear_grouped_t3(ctypes.cast(self.arr, ctypes.c_void_p), self.n, self.xd, self.eps,
                                                  self.yd, _ptr(self.ws), self.ws.numel(), _stream(stream)),
                   "bitnet_linear_grouped_t3")
            return
        if self.bits == 1:
            _check(lib().bitnet_linear_grouped_b1(ctypes.cast(self.arr, ctypes.c_void_p), self.n, self.xd, self.eps,
                                                  self.yd, _ptr(self.ws), self.ws.numel(), _stream(stream)),
                   "bitnet_linear_grouped_b1")
            return
        _check(lib().bitnet_linear_grouped(ctypes.cast(self.arr, ctypes.c_void_p), self.n, self.M, self.xd,
                                           self.eps, self.yd, _ptr(self.ws), self.ws.numel(), _stream(stream)),
               "bitnet_linear_grouped")
