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
