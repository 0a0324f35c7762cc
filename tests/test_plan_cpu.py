"""Host logic of the streaming GEMV's launch plan, on the CPU.

bitnet_debug_stream_plan runs the library's own planner for a described
device (148 SMs, 232448 bytes of opt-in shared memory, as on B200) without
touching a GPU.  These tests pin the K bounds the header documents and check
the plan's invariants on seeded random problem sets."""
import numpy as np
import pytest

import bitlinear_bitnet_linear_b200 as bn
from bitlinear_bitnet_linear_b200 import synthetic

SMS, OPTIN = 148, 232448
# largest K with a plan: (bits, M) -> K, and the K step of the format
BOUND = {(2, 1): 48128, (2, 2): 39936, (2, 3): 29696, (2, 4): 29696, (1, 1): 79872, (3, 1): 57600}
STEP = {1: 128, 2: 64, 3: 16}


def row_bytes(K, bits):
    return (K + 79) // 80 * 16 if bits == 3 else K // 8 * bits


def plan(shapes, M, bits=2, prequant=False):
    return bn.bitnet_debug_stream_plan(shapes, M, bits=bits, prequant=prequant, sms=SMS, smem_optin=OPTIN)


@pytest.mark.parametrize("bits,M", sorted(BOUND))
def test_documented_k_bounds(bits, M):
    K = BOUND[(bits, M)]
    p = plan([(K, 64)], M, bits)
    assert p["smem"] <= OPTIN and p["slot_bytes"] >= row_bytes(K, bits)
    with pytest.raises(bn.BitnetError) as ei:
        plan([(K + STEP[bits], 64)], M, bits)
    assert ei.value.status == 5   # BITNET_ERR_UNSUPPORTED


def test_stack_plan_uses_every_sm_and_both_buffers():
    """The 30-layer stack as one grouped call: a long stream over all SMs,
    two activation buffers and two ring slots per warp."""
    mats = synthetic.stack_matrices(30)
    p = plan([(m.K, m.N) for m in mats], 1)
    assert p["grid"] == SMS and p["nxb"] == 2 and p["nslots"] == 2
    assert p["smem"] <= OPTIN


def _check_invariants(shapes, M, bits, prequant, p):
    assert 1 <= p["grid"] <= SMS
    assert p["smem"] <= OPTIN
    assert p["nxb"] in (1, 2) and p["nslots"] in (1, 2)
    assert p["slot_bytes"] % 128 == 0
    assert p["slot_bytes"] >= max(row_bytes(K, bits) for K, _ in shapes)
    MT = 1 if M <= 1 else (2 if M <= 2 else 4)
    for (K, N), rc, task in zip(shapes, p["rows"], p["task"]):
        assert 1 <= rc <= N
        assert rc * row_bytes(K, bits) <= p["slot_bytes"]       # a chunk fits one slot
        if bits == 3:
            assert task == 9 and (rc < 4 or rc % 4 == 0)
        elif MT == 1 and not prequant:
            lane_task = task - (5 if bits == 1 else 0)            # lane-group tasks 0..3
            assert lane_task in (0, 1, 2, 3)
            assert rc % {0: 8, 1: 4, 2: 2, 3: 1}[lane_task] == 0
        else:
            unit = {1: 4, 2: 2, 4: 1}[MT]                         # whole-warp task
            assert task == 4 and (rc < unit or rc % unit == 0)


@pytest.mark.parametrize("seed", range(40))
def test_random_plans(seed):
    rng = np.random.default_rng(seed)
    bits = int(rng.choice([1, 2, 2, 2, 3]))
    M = int(rng.integers(1, 5)) if bits == 2 else 1
    prequant = bool(bits == 2 and rng.random() < 0.25)
    count = int(rng.choice([1, 2, 3, 7, 30, 210, 256]))
    kmax = BOUND[(bits, M)] * 5 // 4
    step = 64 if bits != 1 else 128
    if bits == 3:
        step = 16
    shapes = [(int(rng.integers(1, kmax // step + 1)) * step, int(rng.integers(1, 30000))) for _ in range(count)]
    fits = max(K for K, _ in shapes) <= BOUND[(bits, M)]
    if fits:
        _check_invariants(shapes, M, bits, prequant, plan(shapes, M, bits, prequant))
    else:
        with pytest.raises(bn.BitnetError) as ei:
            plan(shapes, M, bits, prequant)
        assert ei.value.status == 5


def test_rejects_bad_arguments():
    with pytest.raises(bn.BitnetError) as ei:
        plan([(100, 8)], 1)          # K % 16 != 0
    assert ei.value.status == 2
    with pytest.raises(bn.BitnetError) as ei:
        plan([(256, 8)], 5)          # M above the GEMV's 4 tokens
    assert ei.value.status == 5
    with pytest.raises(bn.BitnetError) as ei:
        plan([(256, 8)] * 257, 1)    # more problems than a grouped call takes
    assert ei.value.status == 2
