"""Host-side parts of bench.py that need no GPU: the reference arm (the
oracle on the host cores) and its row-split harness."""
import json
import os
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.join(ROOT, "oracle"))

import bench  # noqa: E402
import oracle  # noqa: E402


def test_row_split_reproduces_single_thread_forward():
    """Splitting the output rows over threads computes, for every row, the
    oracle's own single-threaded result (bit for bit), ragged split included."""
    oracle.build()
    rng = np.random.default_rng(5)
    K, N = 272, 101
    Wq = rng.integers(-1, 2, (N, K), dtype=np.int8)
    x = rng.standard_normal((1, K)).astype(np.float32)
    gain = np.ones(K, np.float32)
    one = bench._OracleRows(oracle, 1)
    many = bench._OracleRows(oracle, 4)
    try:
        y1 = one(x, Wq, 0.37, gain)
        y4 = many(x, Wq, 0.37, gain)
    finally:
        many.close()
    assert y1.shape == (1, N) and y4.shape == (1, N)
    assert np.array_equal(y1.view(np.uint32), y4.view(np.uint32))


def _run(args, env_extra=None):
    env = dict(os.environ)
    env.pop("RANK", None)
    env.pop("WORLD_SIZE", None)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                          env=env, cwd=ROOT, timeout=600)


def test_reference_arm_prints_one_contract_line():
    r = _run(["--impl", "reference", "--steps", "1", "--warmup", "3"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "GB/s"
    assert d["higher_is_better"] is True and d["n_gpus"] == 1
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["cpu_baseline"]["cores"] == bench.host_cores()
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_without_work():
    r = _run(["--impl", "reference", "--steps", "1", "--warmup", "3"], {"RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_hbm_gate_leg_host_logic(monkeypatch):
    """The gate leg's pool sizing, byte accounting and call pattern, run on
    the CPU against a stand-in for the library binding (no kernels)."""
    import contextlib
    import types

    import torch

    from bitlinear_bitnet_linear_b200 import synthetic

    monkeypatch.setattr(torch.cuda, "stream", lambda s: contextlib.nullcontext())
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    monkeypatch.setattr(bench, "GATE_SHAPES", [(256, 512), (512, 256), (64, 64)])
    monkeypatch.setattr(bench, "L2_BYTES", 40_000)
    seen = {"single": [], "grouped": []}

    def linear(x, Wp, g, N=None, rms_gain=None, rms_eps=1e-5, y=None, ws=None):
        assert x.shape == (1, Wp.shape[1] * 4) and y.shape == (1, N) and Wp.shape[0] == N
        assert rms_gain.shape == (x.shape[1],)
        seen["single"].append(Wp.data_ptr())

    class Grouped:
        def __init__(self, probs, rms_eps=1e-5, ws=None):
            assert 1 <= len(probs) <= 256
            self.probs = probs

        def __call__(self, stream=None):
            seen["grouped"].append(len(self.probs))

    fake = types.SimpleNamespace(
        bitnet_quant_weights=lambda W: (torch.zeros(W.shape, dtype=torch.int8), torch.ones(1)),
        bitnet_pack=lambda Wq: torch.zeros((Wq.shape[0], Wq.shape[1] // 4), dtype=torch.uint8),
        bitnet_linear=linear, GroupedCall=Grouped,
        new_workspace=lambda n, dev=None: torch.empty(n, dtype=torch.uint8),
        bitnet_workspace_bytes=lambda M, K, N: 256, bitnet_get_error=lambda ws: 0)

    def capture(fn):
        fn()
        return fn

    def time_graph(gr, steps, warm, sample_clocks=False):
        gr()
        return 0.5, 0.5, None

    out = bench.hbm_gate_legs(fake, synthetic, torch.device("cpu"), None, capture, time_graph, 1, {})
    shapes = out["shapes"]
    assert [(e["K"], e["N"]) for e in shapes] == bench.GATE_SHAPES
    for e in shapes:
        wbytes = e["N"] * e["K"] // 4
        # at least 3x the (stand-in) L2 in distinct copies, within [8, 240]
        assert e["copies"] == min(240, max(8, -(-3 * bench.L2_BYTES // wbytes)))
        assert e["bytes_per_call"] == wbytes + 2 * e["K"] + 2 * e["N"] + 4
        for form in ("single", "grouped"):
            us = e[form]["us_per_call"]
            assert abs(us - 500.0 / e["copies"]) < 1e-2
            assert e[form]["value"] == round(e["copies"] * e["bytes_per_call"] / 0.5e-3 / 1e9, 2)
    # single launches walk distinct copies (two passes per shape: capture and time)
    n0 = shapes[0]["copies"]
    assert len(set(seen["single"][:n0])) == n0
    assert seen["grouped"] == [e["copies"] for e in shapes for _ in range(2)]


def test_prefill_cpu_baseline_line():
    """The oracle's prefill rate: an M-slice, labelled extrapolated, with the
    all-cores form when the host has more than one core."""
    d = bench.prefill_cpu_baseline(seconds=0.3, m_slice=2)
    assert d["kind"] == "oracle" and d["unit"] == "TOPS" and d["cores"] == 1
    assert d["extrapolated"] is True and d["value"] > 0
    if bench.host_cores() > 1:
        assert d["all_cores"]["cores"] == bench.host_cores() and d["all_cores"]["value"] > 0
