#!/usr/bin/env python
"""BitLinear benchmark on B200.

Default workload (N = 1): decode, M = 1 token, through the BitLinear calls
of a 30-layer BitNet-b1.58-style stack (hidden 2560, FFN 6912): per layer
Q, K, V, O (2560 -> 2560), up, gate (2560 -> 6912) and down (6912 -> 2560),
i.e. the three decode GEMV shapes 2560x2560, 2560x6912 and 6912x2560.  One
step = one token through all 210 calls (fused RMSNorm gain -> absmax int8
quantise -> packed-ternary GEMV -> rescale, bf16 in / bf16 out); the packed
weights (594.7 MB) are larger than L2, so every step streams them from HBM.

value = algorithmic bytes per step (packed weights + x read + y written)
        / device time per step, in GB/s, summed over ranks.
A secondary "prefill" object reports the tensor-core GEMM at M = 4096,
K = 2560, N = 6912 in int8 TOPS (L2 flushed between timed iterations).

Multi-GPU: one process per GPU (torchrun); each rank decodes its own token
stream through its own copy of the stack (data-parallel replicas, no
data-path collective); NCCL only carries the barrier and the max-time
reduction.

--impl reference times the CPU oracle (test infrastructure) on the host cores
on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "BitLinear decode GEMV HBM GB/s (% of peak); prefill GEMM int8 TOPS (% peak)"
# DRAM bytes (read + write) per launch from one ncu capture of each kernel as
# it stands (profiles/); set to None whenever the kernel changes.
# Decode: 79.60 + 3.28 MB on the 4-layer stack, scaled by weight bytes to 30 layers.
TRAFFIC_DECODE = round((79.602688e6 + 3.279872e6) * 597673800 / 79689840)
TRAFFIC_PREFILL = round(15.035648e6 + 4.606464e6)
WORKLOAD = ("decode GEMV M=1 over the 2560x2560 / 2560x6912 / 6912x2560 BitLinear shapes, "
            "30-layer BitNet-b1.58-style stack (210 calls per token, 594.7 MB packed 2-bit weights)")
NOMINAL_INT8_OVER_BF16 = 2.0        # dense int8 (as fp8) vs dense bf16, nominal B200 ratio


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--sustained-steps", type=int, default=2000,
                    help="also time this many decode steps back to back (0: skip)")
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--layers", type=int, default=30)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-chain", action="store_true")
    ap.add_argument("--prefill-iters", type=int, default=50)
    ap.add_argument("--only", choices=["all", "decode", "prefill"], default="all",
                    help="run one part (for profiling a single kernel on a small case)")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), "measured"
    return 6650.0, 1590.0, "fallback"


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"bitnet_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.25)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i in range(4) if r[i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "samples": len(rows), "reasons": reasons}


# ---------------------------------------------------------------------------
# our implementation
# ---------------------------------------------------------------------------
def run_ours(args):
    import torch
    import torch.distributed as dist

    import bitlinear_bitnet_linear_b200 as bn
    from bitlinear_bitnet_linear_b200 import build, replicas, synthetic

    rank, world, local = replicas.rank_info()
    if world > 1:
        torch.cuda.set_device(local)
        replicas.init("nccl", timeout_s=120, device=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    bn.lib()

    hbm_peak, bf16_peak, peak_src = load_peaks()
    stream = torch.cuda.Stream(device=dev)
    if args.only == "prefill":
        res = run_prefill(args, dev, stream, bf16_peak, peak_src)
        if world > 1:
            dist.destroy_process_group()
        return res if rank == 0 else None
    if args.only == "decode":
        args.no_prefill = True

    # ---- the stack: weights quantised and packed on the device ------------
    mats = synthetic.stack_matrices(args.layers)
    stack = []
    gens = torch.Generator(device=dev)
    with torch.cuda.stream(stream):
        for mt in mats:
            gens.manual_seed(mt.seed)
            W = torch.randn((mt.N, mt.K), generator=gens, device=dev, dtype=torch.float32) * synthetic.W_SIGMA
            Wq, g = bn.bitnet_quant_weights(W)
            Wp = bn.bitnet_pack(Wq)
            del W, Wq
            stack.append((mt.K, mt.N, Wp, g))
    torch.cuda.synchronize()
    gains = {K: synthetic.unit_gain(K).to(dev) for K in {m.K for m in mats}}
    # inputs of one step: one bf16 activation row per call (independent of the rank's replica)
    xs_host = [synthetic.activations(1, K, seed=replicas.replica_seed(i, rank), dtype=torch.bfloat16)
               for i, (K, N, _, _) in enumerate(stack)]
    xs = [x.to(dev) for x in xs_host]
    ys = [torch.empty((1, N), dtype=torch.bfloat16, device=dev) for (K, N, _, _) in stack]
    ws = bn.new_workspace(max(bn.bitnet_workspace_bytes(1, K, N) for (K, N, _, _) in stack), dev)

    bytes_step = sum(N * K // 4 + K * 2 + N * 2 + 4 for (K, N, _, _) in stack)
    calls = len(stack)
    problems = [(x, Wp, g, gains[K], y) for (K, N, Wp, g), x, y in zip(stack, xs, ys)]
    grouped = bn.GroupedCall(problems, rms_eps=1e-5, ws=ws)

    def step():
        grouped()

    def chain_step():
        for (K, N, Wp, g), x, y in zip(stack, xs, ys):
            bn.bitnet_linear(x, Wp, g, N=N, rms_gain=gains[K], rms_eps=1e-5, y=y, ws=ws)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def capture(fn):
        with torch.cuda.stream(stream):
            for _ in range(2):
                fn()
        torch.cuda.synchronize()
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=stream):
            fn()
        torch.cuda.synchronize()
        assert bn.bitnet_get_error(ws) == 0
        return gr

    def time_graph(gr, steps, warm, sample_clocks=False):
        for _ in range(max(3, warm)):
            gr.replay()
        barrier()
        clk = None
        sampler = ClockSampler(dev.index) if sample_clocks else None
        if sampler:
            sampler.start()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        barrier()
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(steps):
                gr.replay()
            e1.record(stream)
        barrier()
        if sampler:
            clk = sampler.stop()
        ms_local = e0.elapsed_time(e1) / steps
        return ms_local, replicas.max_over_ranks(ms_local, dev), clk

    # Ten steps per graph: inside a graph, each step's launch overlaps its
    # weight prefetch with the previous step's tail (programmatic dependent
    # launch); separate graph replays cannot overlap.  Exactly args.steps
    # steps are timed (a one-step graph covers any remainder).
    per_graph = max(1, min(10, args.steps))

    def steps_fn(n):
        def fn():
            for _ in range(n):
                step()
        return fn

    graph = capture(steps_fn(per_graph))
    graph1 = capture(step) if args.steps % per_graph else None

    def time_steps(steps, warm, sample_clocks=False):
        for _ in range(max(3, warm)):
            graph.replay()
        barrier()
        sampler = ClockSampler(dev.index) if sample_clocks else None
        if sampler:
            sampler.start()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        barrier()
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(steps // per_graph):
                graph.replay()
            for _ in range(steps % per_graph):
                graph1.replay()
            e1.record(stream)
        barrier()
        clk = sampler.stop() if sampler else None
        ms_local = e0.elapsed_time(e1) / steps
        return ms_local, replicas.max_over_ranks(ms_local, dev), clk

    ms, ms_max, clk = time_steps(args.steps, args.warmup, sample_clocks=True)
    assert bn.bitnet_get_error(ws) == 0
    # The same steps over a longer run: HBM streaming slows down after a few
    # tens of milliseconds of continuous load on this part.
    sustained = None
    if args.sustained_steps > 0:
        s_ms, s_ms_max, s_clk = time_steps(args.sustained_steps, 3, sample_clocks=True)
        sustained = {"steps": args.sustained_steps, "ms_per_step": round(s_ms_max, 5),
                     "value": round(replicas.whole_job_rate(bytes_step, world, s_ms_max * 1e-3) / 1e9, 2),
                     "unit": "GB/s", "clocks": s_clk}
    value = replicas.whole_job_rate(bytes_step, world, ms_max * 1e-3) / 1e9
    per_rank = bytes_step / (ms * 1e-3) / 1e9

    # ---- the same 210 calls as a dependent chain of separate launches ------
    chain = None
    if not args.no_chain:
        cgraph = capture(chain_step)
        csteps = max(20, args.steps // 10)
        cms, cms_max, _ = time_graph(cgraph, csteps, 3)
        chain = {"value": round(world * bytes_step / (cms_max * 1e-3) / 1e9, 2), "unit": "GB/s",
                 "ms_per_step": round(cms_max, 4), "us_per_call": round(cms_max * 1e3 / calls, 3),
                 "steps": csteps, "launches_per_step": calls,
                 "what": "each of the 210 calls its own bitnet_linear launch, in stream order (each waits for "
                         "the previous), programmatic dependent launch, one CUDA graph per step"}
        del cgraph

    # ---- the feed-forward chain: each layer's down projection consumes the
    # ReLU^2 gate of its up/gate outputs and updates the residual stream ----
    ffn = None
    if not args.no_chain:
        layers = len(stack) // 7
        hidden = stack[0][0]
        h = synthetic.activations(1, hidden, seed=replicas.replica_seed(10_000, rank),
                                  dtype=torch.bfloat16).to(dev)
        f_calls, f_bytes = [], 0
        for l in range(layers):
            (Ku, Nu, Wu, gu), (Kg, Ng, Wg, gg), (Kd, Nd, Wd, gd) = stack[7 * l + 4: 7 * l + 7]
            yu = torch.empty((1, Nu), dtype=torch.bfloat16, device=dev)
            yg = torch.empty((1, Ng), dtype=torch.bfloat16, device=dev)
            upgate = bn.GroupedCall([(h, Wu, gu, gains[Ku], yu), (h, Wg, gg, gains[Kg], yg)], rms_eps=1e-5)
            f_calls.append((upgate, yg, yu, Wd, gd, gains[Kd], Nd))
            f_bytes += (Nu * Ku + Ng * Kg + Nd * Kd) // 4 + Ku * 2 + (Nu + Ng) * 2 * 2 + Kd * 2 + Nd * 2 * 2 + 12

        def ffn_step():
            for upgate, yg, yu, Wd, gd, gaind, Nd in f_calls:
                upgate()
                bn.bitnet_linear_relu2(yg, yu, Wd, gd, N=Nd, rms_gain=gaind, rms_eps=1e-5, resid=h, y=h, ws=ws)

        fgraph = capture(ffn_step)
        fsteps = max(20, args.steps // 10)
        fms, fms_max, _ = time_graph(fgraph, fsteps, 3)
        assert bn.bitnet_get_error(ws) == 0
        ffn = {"value": round(world * f_bytes / (fms_max * 1e-3) / 1e9, 2), "unit": "GB/s",
               "ms_per_step": round(fms_max, 4), "us_per_layer": round(fms_max * 1e3 / layers, 3),
               "steps": fsteps, "launches_per_step": 2 * layers, "bytes_per_step": f_bytes,
               "what": "per layer: up|gate as one grouped launch on the residual stream, then the down "
                       "projection with the ReLU^2 gate fused into its quantiser and the residual added in "
                       "its epilogue (bitnet_linear_relu2, in place); 60 dependent launches, one CUDA graph"}
        del fgraph

    # ---- BitNet b1: the same stack with binary weights, 1 bit per weight ----
    b1 = None
    if not args.no_chain:
        b1_stack = []
        with torch.cuda.stream(stream):
            for mt in mats:
                gens.manual_seed(mt.seed)
                W = torch.randn((mt.N, mt.K), generator=gens, device=dev, dtype=torch.float32) * synthetic.W_SIGMA
                Wb, beta = bn.bitnet_quant_weights_b1(W)
                b1_stack.append((bn.bitnet_pack_b1(Wb), beta))
                del W, Wb
        torch.cuda.synchronize()
        b1_call = bn.GroupedCall([(x, Wp1, beta, gains[K], y) for (K, N, _, _), (Wp1, beta), x, y
                                  in zip(stack, b1_stack, xs, ys)], rms_eps=1e-5, ws=ws, bits=1)

        def b1_steps(n):
            def fn():
                for _ in range(n):
                    b1_call()
            return fn

        b1_bytes = sum(N * K // 8 + K * 2 + N * 2 + 4 for (K, N, _, _) in stack)
        b1_graph = capture(b1_steps(per_graph))
        bsteps = (max(20, args.steps // 2) // per_graph) * per_graph
        bms, bms_max, _ = time_graph(b1_graph, bsteps // per_graph, 3)
        bms, bms_max = bms / per_graph, bms_max / per_graph
        assert bn.bitnet_get_error(ws) == 0
        b1 = {"value": round(world * b1_bytes / (bms_max * 1e-3) / 1e9, 2), "unit": "GB/s",
              "ms_per_step": round(bms_max, 5), "tokens_per_s": round(world * 1e3 / bms_max, 1),
              "bytes_per_step": b1_bytes, "steps": bsteps,
              "what": "the 210-call stack with BitNet b1 weights (sign, absmean scale, 1 bit per weight, "
                      "297 MB), one grouped launch per token (bitnet_linear_grouped_b1), CUDA graphs of "
                      f"{per_graph} steps"}
        del b1_graph, b1_call, b1_stack

    # ---- base-3: the same ternary stack at five weights per byte ------------
    t3 = None
    if not args.no_chain:
        t3_packed = []
        with torch.cuda.stream(stream):
            for (K, N, Wp, g) in stack:
                t3_packed.append(bn.bitnet_pack_t3(bn.bitnet_unpack(Wp, K)))
        torch.cuda.synchronize()
        t3_call = bn.GroupedCall([(x, Wp3, g, gains[K], y) for (K, N, _, g), Wp3, x, y
                                  in zip(stack, t3_packed, xs, ys)], rms_eps=1e-5, ws=ws, bits=3)

        def t3_steps(n):
            def fn():
                for _ in range(n):
                    t3_call()
            return fn

        t3_bytes = sum(N * bn.bitnet_t3_row_bytes(K) + K * 2 + N * 2 + 4 for (K, N, _, _) in stack)
        t3_graph = capture(t3_steps(per_graph))
        tsteps = (max(20, args.steps // 2) // per_graph) * per_graph
        tms, tms_max, _ = time_graph(t3_graph, tsteps // per_graph, 3)
        tms, tms_max = tms / per_graph, tms_max / per_graph
        assert bn.bitnet_get_error(ws) == 0
        t3 = {"value": round(world * t3_bytes / (tms_max * 1e-3) / 1e9, 2), "unit": "GB/s",
              "ms_per_step": round(tms_max, 5), "tokens_per_s": round(world * 1e3 / tms_max, 1),
              "bytes_per_step": t3_bytes, "steps": tsteps,
              "what": "the same ternary stack packed base-3 (five weights per byte, 1.6 bits per weight), one "
                      "grouped launch per token (bitnet_linear_grouped_t3), digits decoded in registers"}
        del t3_graph, t3_call, t3_packed

    # ---- e2e: host buffers, through the public API, no graph ----------------
    e2e = None
    if not args.no_e2e:
        h2d = sum(x.numel() * 2 for x in xs_host)
        d2h = sum(y.numel() * 2 for y in ys)
        x_pin = torch.cat([x.reshape(-1) for x in xs_host]).pin_memory()
        y_pin = torch.empty(sum(y.numel() for y in ys), dtype=torch.bfloat16).pin_memory()
        # two device buffer sets, so step t's kernel overlaps the H2D copy of
        # step t + 1 and the D2H copy of step t - 1 (copy streams, events);
        # every step still moves its own inputs and result across the bus
        x_dev = [torch.empty_like(x_pin, device=dev) for _ in range(2)]
        y_dev = [torch.empty(y_pin.numel(), dtype=torch.bfloat16, device=dev) for _ in range(2)]
        xo, yo = [], []
        o = 0
        for x in xs_host:
            xo.append((o, x.shape[1]))
            o += x.numel()
        o = 0
        for y in ys:
            yo.append((o, y.shape[1]))
            o += y.numel()
        ecalls = []
        for bsel in range(2):
            xviews = [x_dev[bsel][a:a + k].view(1, k) for a, k in xo]
            yviews = [y_dev[bsel][a:a + n].view(1, n) for a, n in yo]
            eproblems = [(x, Wp, g, gains[K], y) for (K, N, Wp, g), x, y in zip(stack, xviews, yviews)]
            ecalls.append(bn.GroupedCall(eproblems, rms_eps=1e-5, ws=ws))
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_k = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def e2e_run(n):
            for i in range(n):
                bsel = i & 1
                s_in.wait_event(ev_k[bsel])                 # x buffer read by the kernel two steps back
                with torch.cuda.stream(s_in):
                    x_dev[bsel].copy_(x_pin, non_blocking=True)
                ev_in[bsel].record(s_in)
                stream.wait_event(ev_in[bsel])
                stream.wait_event(ev_out[bsel])            # y buffer copied out two steps back
                ecalls[bsel](stream)
                ev_k[bsel].record(stream)
                s_out.wait_event(ev_k[bsel])
                with torch.cuda.stream(s_out):
                    y_pin.copy_(y_dev[bsel], non_blocking=True)
                ev_out[bsel].record(s_out)

        e2e_steps = max(10, min(500, args.steps // 4))
        e2e_run(4)
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        e2e_run(e2e_steps)
        e1.record(s_out)
        barrier()
        ems = replicas.max_over_ranks(e0.elapsed_time(e1) / e2e_steps, dev)
        e2e = {"value": round(replicas.whole_job_rate(bytes_step, world, ems * 1e-3) / 1e9, 2), "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(ems, 4),
               "path": "python binding (prepared GroupedCall) -> C ABI bitnet_linear_grouped (210 problems); "
                       "per step one pinned-host copy of all x in and one of all y out, on copy streams that "
                       "overlap the neighbouring steps' kernels (two device buffer sets), no graph"}

    # ---- prefill GEMM (secondary) ------------------------------------------
    prefill = None
    if not args.no_prefill:
        prefill = run_prefill(args, dev, stream, bf16_peak, peak_src)

    # ---- CPU oracle baseline (rank 0 at N = 1 only) --------------------------
    cpu = None
    if not args.no_cpu_baseline and world == 1 and rank == 0:
        cpu = cpu_baseline(layers_sample=1)
        if prefill is not None:
            prefill["cpu_baseline"] = prefill_cpu_baseline()

    # ---- single-matrix HBM gates: each shape at M = 1 over a pool of distinct
    # weight copies (together well beyond L2), as separate launches and as
    # one grouped launch.  Last, so that nothing else depends on it; a
    # failure here is reported in its own key.  One GPU only: a failure on
    # one rank must not leave the ranks' collectives out of step. -----------
    gates = None
    if not args.no_chain and world == 1:
        try:
            gates = hbm_gate_legs(bn, synthetic, dev, stream, capture, time_graph, world, gains)
            torch.cuda.synchronize()
        except Exception as e:   # noqa: BLE001 - the headline line must still print
            gates = {"error": repr(e)[:300]}

    del graph, graph1
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return None

    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": round(ms_max, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8 x ternary(2-bit) -> int32",
        "data": "synthetic (seeded N(0,0.02) latent weights, N(0,1) activations with 1% x20 outliers)",
        "config": {"workload": WORKLOAD, "tokens_per_step": world, "calls_per_step": calls,
                   "bytes_per_step_per_gpu": bytes_step,
                   "l2": "inputs larger than L2 (594.7 MB of packed weights per step per GPU)",
                   "parallelism": f"dp{world} (independent replicas, no data-path collective)",
                   "launch": "the step's 210 independent calls as one grouped launch (bitnet_linear_grouped); "
                             "CUDA graphs of 10 steps, each launch waiting on the previous one (programmatic "
                             "dependent launch)"},
        "tokens_per_s": round(world * 1e3 / ms_max, 1),
        "roofline": {"bound": "hbm", "kernel": "gemv_stream_kernel<1,256,15> (grouped fused quantise + GEMV, per-warp weight rings)",
                     "achieved": round(per_rank, 2), "peak": hbm_peak, "unit": "GB/s",
                     "frac": round(per_rank / hbm_peak, 4), "peak_source": f"{peak_src} HBM copy bandwidth",
                     "frac_of_8TBs_datasheet": round(per_rank / 8000.0, 4),
                     "traffic": TRAFFIC_DECODE,
                     "note": "one launch of this kernel per step; achieved = algorithmic bytes per launch / "
                             "mean launch duration"},
        "gpu_launches": args.steps,
        "clocks": clk,
    }
    if sustained is not None:
        out["sustained"] = sustained
    if e2e is not None:
        out["e2e"] = e2e
    if chain is not None:
        out["decode_chain"] = chain
    if ffn is not None:
        out["ffn_chain"] = ffn
    if b1 is not None:
        out["b1_decode"] = b1
    if t3 is not None:
        out["t3_decode"] = t3
    if gates is not None:
        out["hbm_gates"] = gates
    # every HBM-bound leg against the same measured copy bandwidth, per GPU
    for key in ("decode_chain", "ffn_chain", "b1_decode", "t3_decode"):
        if key in out:
            out[key]["frac_of_hbm_peak"] = round(out[key]["value"] / world / hbm_peak, 4)
    for e in (gates or {}).get("shapes", []):
        for form in ("single", "grouped"):
            e[form]["frac_of_hbm_peak"] = round(e[form]["value"] / world / hbm_peak, 4)
    if prefill is not None:
        out["prefill"] = prefill
    if cpu is not None:
        out["cpu_baseline"] = cpu
    return out


L2_BYTES = 126 * 2 ** 20
GATE_SHAPES = [(8192, 28672), (28672, 8192), (2560, 2560), (2560, 6912), (6912, 2560)]   # (K, N)


def hbm_gate_legs(bn, synthetic, dev, stream, capture, time_graph, world, gains):
    """Decode (M = 1) over one shape at a time.  Each shape gets a pool of
    distinct copies of one packed matrix, at least 3x L2 in total (at most
    240 copies), with its own bf16 activation row and output per copy:
    - single: one bitnet_linear launch per copy, in stream order, one CUDA
      graph per pass over the pool;
    - grouped: the whole pool as one bitnet_linear_grouped launch.
    Bytes per call: N K / 4 + 2 K + 2 N + 4."""
    import torch
    res = []
    for K, N in GATE_SHAPES:
        wbytes = N * K // 4
        copies = int(min(240, max(8, -(-3 * L2_BYTES // wbytes))))
        gen = torch.Generator(device=dev).manual_seed(7000 + K + N)
        with torch.cuda.stream(stream):
            W = torch.randn((N, K), generator=gen, device=dev, dtype=torch.float32) * synthetic.W_SIGMA
            Wq, g = bn.bitnet_quant_weights(W)
            Wp0 = bn.bitnet_pack(Wq)
            del W, Wq
            pool = [Wp0.clone() for _ in range(copies)]
        torch.cuda.synchronize()
        del Wp0
        gain = gains[K] if K in gains else synthetic.unit_gain(K).to(dev)
        xs = [synthetic.activations(1, K, seed=8000 + i, dtype=torch.bfloat16).to(dev) for i in range(copies)]
        ys = [torch.empty((1, N), dtype=torch.bfloat16, device=dev) for _ in range(copies)]
        ws = bn.new_workspace(bn.bitnet_workspace_bytes(1, K, N), dev)
        call_bytes = wbytes + 2 * K + 2 * N + 4

        def single():
            for Wp, x, y in zip(pool, xs, ys):
                bn.bitnet_linear(x, Wp, g, N=N, rms_gain=gain, rms_eps=1e-5, y=y, ws=ws)

        grouped = bn.GroupedCall([(x, Wp, g, gain, y) for Wp, x, y in zip(pool, xs, ys)], rms_eps=1e-5, ws=ws)
        entry = {"K": K, "N": N, "copies": copies, "pool_mb": round(copies * wbytes / 1e6, 1),
                 "bytes_per_call": call_bytes}
        for name, fn in (("single", single), ("grouped", grouped)):
            gr = capture(fn)
            ms, ms_max, _ = time_graph(gr, 20, 3)
            assert bn.bitnet_get_error(ws) == 0
            entry[name] = {"value": round(world * copies * call_bytes / (ms_max * 1e-3) / 1e9, 2), "unit": "GB/s",
                           "us_per_call": round(ms_max * 1e3 / copies, 3)}
            del gr
        res.append(entry)
        del pool, xs, ys, grouped
        torch.cuda.synchronize()
    return {"what": "M = 1 BitLinear (bf16 x, unit RMSNorm gain, bf16 y) per shape over a pool of distinct "
                    "weight copies of at least 3x L2; single = one bitnet_linear launch per call in stream "
                    "order, grouped = the pool as one bitnet_linear_grouped launch; CUDA graphs, 20 passes",
            "shapes": res}


def run_prefill(args, dev, stream, bf16_peak, peak_src):
    """Tensor-core GEMM at M = 4096, K = 2560, N = 6912 (bf16 x, fused unit
    RMSNorm gain, bf16 y).  Each iteration is timed alone with L2 flushed."""
    import torch

    import bitlinear_bitnet_linear_b200 as bn
    from bitlinear_bitnet_linear_b200 import synthetic

    M, K, N = 4096, 2560, 6912
    g = torch.Generator(device=dev)
    g.manual_seed(4242)
    with torch.cuda.stream(stream):
        W = torch.randn((N, K), generator=g, device=dev) * synthetic.W_SIGMA
        Wq, gam = bn.bitnet_quant_weights(W)
        Wp = bn.bitnet_pack(Wq)
        del W, Wq
    x = synthetic.activations(M, K, seed=4243).to(dev)
    gain = synthetic.unit_gain(K).to(dev)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    ws = bn.new_workspace(bn.bitnet_workspace_bytes(M, K, N), dev)
    xq, sc, xsum = bn.bitnet_quant_act(x, gain)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()

    def timed(fn, iters):
        ts = []
        for _ in range(iters):
            with torch.cuda.stream(stream):
                flush.fill_(1)
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                fn()
                b.record(stream)
            b.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    with torch.cuda.stream(stream):
        for _ in range(3):
            bn.bitnet_linear(x, Wp, gam, rms_gain=gain, y=y, ws=ws, path=bn.PATH_TC)
    torch.cuda.synchronize()
    full_ms = timed(lambda: bn.bitnet_linear(x, Wp, gam, rms_gain=gain, y=y, ws=ws, path=bn.PATH_TC),
                    args.prefill_iters)
    gemm_ms = timed(lambda: bn.bitnet_linear_q(xq, sc, Wp, gam, x_sum=xsum, y=y, ws=ws, path=bn.PATH_TC),
                    args.prefill_iters)
    assert bn.bitnet_get_error(ws) == 0
    ops = 2.0 * M * N * K
    peak = bf16_peak * NOMINAL_INT8_OVER_BF16
    # black-box vendor int8 GEMM on the same box, for context
    cublas = None
    try:
        a8 = torch.randint(-127, 128, (8192, 8192), dtype=torch.int8, device=dev)
        b8 = torch.randint(-127, 128, (8192, 8192), dtype=torch.int8, device=dev).t()
        for _ in range(3):
            torch._int_mm(a8, b8)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(10):
            torch._int_mm(a8, b8)
        e1.record()
        torch.cuda.synchronize()
        cublas = round(2 * 8192 ** 3 / (e0.elapsed_time(e1) / 10 * 1e-3) / 1e12, 1)
        del a8, b8
    except Exception as exc:  # noqa: BLE001
        cublas = f"unavailable: {type(exc).__name__}"
    gemm_tops = ops / (gemm_ms * 1e-3) / 1e12
    return {
        "metric": "prefill GEMM int8 TOPS", "unit": "TOPS",
        "config": {"workload": "prefill GEMM M=4096, K=2560, N=6912, bf16 x with fused unit-gain RMSNorm, bf16 y",
                   "l2": "flushed (256 MB write) before every timed iteration", "iters": args.prefill_iters},
        "value": round(ops / (full_ms * 1e-3) / 1e12, 2), "ms": round(full_ms, 4),
        "gemm_only_value": round(gemm_tops, 2), "gemm_only_ms": round(gemm_ms, 4),
        "roofline": {"bound": "tensor", "kernel": "tc_gemm_persistent_kernel<128,8,2,2> (tcgen05 kind::i8 TS form, 256x128 tiles, A expanded into TMEM, three rotating TMEM accumulator slots)", "achieved": round(gemm_tops, 2),
                     "peak": round(peak, 1), "unit": "TFLOP/s",
                     "frac": round(gemm_tops / peak, 4),
                     "peak_source": f"{peak_src} dense bf16 (burst) x {NOMINAL_INT8_OVER_BF16} nominal int8/bf16 ratio",
                     "frac_of_4500_datasheet": round(gemm_tops / 4500.0, 4), "traffic": TRAFFIC_PREFILL},
        "cublas_int8_8192cube_tops": cublas,
        "tokens_per_s": round(M / (full_ms * 1e-3), 1),
    }


# ---------------------------------------------------------------------------
# CPU oracle (test infrastructure) timed on the host cores
# ---------------------------------------------------------------------------
def _oracle_decode_setup(seed0: int):
    """One layer's seven decode calls, prepared for the oracle (weights
    quantised by the oracle itself)."""
    sys.path.insert(0, os.path.join(ROOT, "oracle"))
    import numpy as np

    import oracle
    from bitlinear_bitnet_linear_b200 import synthetic

    oracle.build()
    mats = synthetic.layer_matrices(0)
    prepared = []
    for mt in mats:
        W = synthetic.latent_weights(mt.N, mt.K, mt.seed).numpy()
        Wq, g = oracle.quant_weights(W)
        prepared.append((mt.K, mt.N, Wq, g))
    gain = {K: np.ones(K, np.float32) for K in {m.K for m in mats}}
    xs = [synthetic.activations(1, K, seed=seed0 + i).float().numpy() for i, (K, _, _, _) in enumerate(prepared)]
    return oracle, prepared, gain, xs


class _OracleRows:
    """Runs the oracle's whole forward (quantise, contract, rescale) for one
    call split by output rows over `threads` host threads.  The oracle is C
    called through ctypes, which releases the GIL, so the slices run in
    parallel; each slice is the oracle's own computation for those rows."""

    def __init__(self, oracle, threads: int):
        from concurrent.futures import ThreadPoolExecutor
        self.oracle = oracle
        self.threads = threads
        self.pool = ThreadPoolExecutor(max_workers=threads) if threads > 1 else None

    def __call__(self, x, Wq, g, gain):
        if self.pool is None:
            return self.oracle.bitlinear(x, Wq, g, gain, 1e-5)[0]
        N = Wq.shape[0]
        cuts = [N * t // self.threads for t in range(self.threads + 1)]
        futs = [self.pool.submit(self.oracle.bitlinear, x, Wq[a:b], g, gain, 1e-5)
                for a, b in zip(cuts[:-1], cuts[1:]) if b > a]
        import numpy as np
        return np.concatenate([f.result()[0] for f in futs], axis=1)

    def close(self):
        if self.pool is not None:
            self.pool.shutdown()


def host_cores() -> int:
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)


def cpu_baseline(layers_sample: int = 1, seconds: float = 10.0):
    """Oracle quantise + contract + rescale for every call of one decode step,
    on a bounded sample: one layer's seven matrices, repeated for about
    `seconds` of CPU time, single-threaded; then the same over all host
    cores (rows split across threads).  The per-step figure scales the
    sample's bytes and time (all layers have the same shapes)."""
    import numpy as np

    oracle, prepared, gain, xs = _oracle_decode_setup(777)
    one = _OracleRows(oracle, 1)

    def run(fn, budget):
        t0 = time.perf_counter()
        nbytes, reps = 0, 0
        while True:
            for (K, N, Wq, g), x in zip(prepared, xs):
                fn(x, Wq, g, gain[K])
                nbytes += N * K // 4 + K * 2 + N * 2 + 4
            reps += 1
            if time.perf_counter() - t0 > budget and reps >= layers_sample:
                break
        return nbytes, reps, time.perf_counter() - t0

    nbytes, reps, dt = run(one, seconds)
    out = {"value": round(nbytes / dt / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
           "sample": f"{reps} x one layer's 7 decode calls (M=1, K x N = 2560x2560 x4, 2560x6912 x2, 6912x2560), "
                     f"same algorithmic-byte accounting, {dt:.1f} s of single-threaded scalar C",
           "ms_per_layer": round(dt * 1e3 / reps, 2)}
    cores = host_cores()
    if cores > 1:
        many = _OracleRows(oracle, cores)
        try:
            # the row split computes exactly the single-threaded result
            (K, N, Wq, g), x = prepared[0], xs[0]
            assert np.array_equal(many(x, Wq, g, gain[K]).view(np.uint32), one(x, Wq, g, gain[K]).view(np.uint32))
            mbytes, mreps, mdt = run(many, seconds / 2)
        finally:
            many.close()
        out["all_cores"] = {"value": round(mbytes / mdt / 1e9, 4), "unit": "GB/s", "cores": cores,
                            "threads": cores, "ms_per_layer": round(mdt * 1e3 / mreps, 2),
                            "sample": f"{mreps} x the same layer, output rows split over {cores} threads "
                                      f"(sched_getaffinity), {mdt:.1f} s"}
    return out


def prefill_cpu_baseline(seconds: float = 6.0, m_slice: int = 8):
    """The oracle on the prefill workload (M = 4096, K = 2560, N = 6912,
    unit RMSNorm gain), timed on an M-slice of m_slice tokens: the oracle's
    forward costs the same per token, so its TOPS carry over to the full M
    (reported as extrapolated).  Single-threaded, then with the output rows
    split over all host cores."""
    sys.path.insert(0, os.path.join(ROOT, "oracle"))
    import numpy as np

    import oracle
    from bitlinear_bitnet_linear_b200 import synthetic

    oracle.build()
    K, N = 2560, 6912
    Wq, g = oracle.quant_weights(synthetic.latent_weights(N, K, seed=4242).numpy())
    x = synthetic.activations(m_slice, K, seed=4243).float().numpy()
    gain = np.ones(K, np.float32)

    def run(fn, budget):
        t0 = time.perf_counter()
        reps = 0
        while True:
            fn(x, Wq, g, gain)
            reps += 1
            if time.perf_counter() - t0 > budget:
                break
        return reps, time.perf_counter() - t0

    ops = 2.0 * m_slice * N * K
    reps, dt = run(_OracleRows(oracle, 1), seconds)
    out = {"value": round(ops * reps / dt / 1e12, 6), "unit": "TOPS", "cores": 1, "kind": "oracle",
           "extrapolated": True,
           "sample": f"{reps} x an M-slice of {m_slice} tokens of the M = 4096 prefill workload, {dt:.1f} s of "
                     f"single-threaded scalar C; the per-token cost is constant, so the rate carries over"}
    cores = host_cores()
    if cores > 1:
        many = _OracleRows(oracle, cores)
        try:
            mreps, mdt = run(many, seconds / 2)
        finally:
            many.close()
        out["all_cores"] = {"value": round(ops * mreps / mdt / 1e12, 6), "unit": "TOPS", "cores": cores,
                            "threads": cores, "sample": f"{mreps} x the same slice, output rows split over "
                                                        f"{cores} threads, {mdt:.1f} s"}
    return out


def run_reference(args):
    """The oracle as the reference arm: one layer's seven decode calls per
    step, output rows split over all host cores."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    oracle, prepared, gain, xs = _oracle_decode_setup(888)
    bytes_sample = sum(N * K // 4 + K * 2 + N * 2 + 4 for (K, N, _, _) in prepared)
    cores = host_cores()
    fn = _OracleRows(oracle, cores)

    def step():
        for (K, N, Wq, g), x in zip(prepared, xs):
            fn(x, Wq, g, gain[K])

    warm = max(3, min(args.warmup, 10))
    try:
        for _ in range(warm):
            step()
        steps = max(1, min(args.steps, 20))
        t0 = time.perf_counter()
        for _ in range(steps):
            step()
        dt = (time.perf_counter() - t0) / steps
    finally:
        fn.close()
    v = bytes_sample / dt / 1e9
    return {"impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": "GB/s", "n_gpus": world,
            "steps": steps, "warmup": warm, "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int8 x ternary -> int32 (scalar C)",
            "data": "synthetic", "config": {"workload": WORKLOAD, "sample": "one layer (7 calls) per step"},
            "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": f"one layer's 7 decode calls per step, scalar C oracle, output rows split "
                                       f"over {cores} host threads"},
            "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    args = parse_args()
    out = run_reference(args) if args.impl == "reference" else run_ours(args)
    if out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
