"""Benchmark of the one-GPU MoE layer forward (router -> permute -> grouped
FFN -> combine).  Default workload: the fine-grained bf16 prefill layer,
N=16384 tokens, d=2048, E=128 experts, top-8, SwiGLU FFN d->768->d, fp32
router with a Zipf-like per-expert bias 1.2*ln(1/rank) (skewed expert loads,
some experts empty); seeded synthetic inputs.  --workload picks another one.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    python bench.py --measure-peak      # dense e4m3 / bf16 matmul peaks of this GPU

One JSON line on rank 0.  ``value`` is whole-job tokens/s from CUDA events on
the launching stream (max over ranks), inputs resident in HBM, L2 flushed
(a 256 MiB write) before every step.  ``e2e`` is the same metric through the
host-buffer entry point (moe_forward_host: pinned H2D of x, the layer, D2H of
y).  ``roofline`` reports the dominant kernel (the fused gate/up SwiGLU grouped
GEMM) against the measured bf16 tensor peak.  ``cpu_baseline`` times the CPU
oracle on a bounded sample of the same workload.  Under torchrun (N > 1) every
rank runs an independent replica of the layer on its own GPU (the layer needs
no exchange between GPUs: weak scaling).

``--impl reference`` times the CPU oracle itself (the reference arm: it is
the plain fp64 restatement of the method), on the host cores, one bounded
token sample per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE layer tokens/s and grouped-GEMM TFLOP/s (% of tensor/HBM roofline), 1 B200"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FLUSH_BYTES = 256 << 20
DEFAULT_WORKLOAD = "bf16_n16384_d2048_e128_k8_f768_swiglu_zipf"
E4M3_PEAK_FILE = os.path.join(ROOT, "profiles", "peak_e4m3_matmul_8192.md")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--measure-peak", action="store_true",
                    help="time dense 8192^3 e4m3 and bf16 matmuls (cuBLASLt through torch) "
                         "and write the e4m3 peak file that the fp8 rooflines divide by")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target CPU time of the oracle baseline sample")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def load_e4m3_peak():
    """The measured dense e4m3 matmul peaks (burst, sustained) in TFLOP/s from
    the committed peak file, or None."""
    if not os.path.exists(E4M3_PEAK_FILE):
        return None
    text = open(E4M3_PEAK_FILE).read()
    vals = {}
    for key in ("e4m3_tflops", "e4m3_tflops_sustained"):
        m = re.search(rf"^{key}:\s*([0-9.eE+]+)\s*$", text, re.M)
        if not m:
            return None
        vals[key] = float(m.group(1))
    return vals


def measure_peak(steps_burst: int = 10, sustain_s: float = 4.0):
    """Dense matmul peaks of this GPU through torch (cuBLASLt): e4m3 x e4m3 ->
    bf16 with unit fp32 scales (torch._scaled_mm) and bf16 x bf16, both
    8192^3 (2 * 8192^3 FLOP).  Burst = the best of `steps_burst` single runs
    (CUDA events, after warm-up); sustained = the mean over back-to-back runs
    for `sustain_s` seconds, under the power cap.  SM clocks are sampled
    meanwhile.  Writes E4M3_PEAK_FILE and prints one JSON line."""
    import torch
    n = 8192
    flop = 2.0 * n * n * n
    torch.manual_seed(0)
    a8 = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn)
    b8 = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn).t()  # column-major operand
    one = torch.ones((), device="cuda")
    a16 = torch.randn(n, n, device="cuda", dtype=torch.bfloat16)
    b16 = torch.randn(n, n, device="cuda", dtype=torch.bfloat16)
    runs = {
        "e4m3": lambda: torch._scaled_mm(a8, b8, scale_a=one, scale_b=one, out_dtype=torch.bfloat16),
        "bf16": lambda: torch.matmul(a16, b16),
    }
    out = {}
    with ClockSampler(torch.cuda.current_device()) as clk:
        for name, f in runs.items():
            for _ in range(5):
                f()
            torch.cuda.synchronize()
            best = float("inf")
            for _ in range(steps_burst):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                f()
                e1.record()
                e1.synchronize()
                best = min(best, e0.elapsed_time(e1))
            # sustained: launch in batches of 20 until sustain_s has passed
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            count = 0
            t0 = time.perf_counter()
            e0.record()
            while time.perf_counter() - t0 < sustain_s:
                for _ in range(20):
                    f()
                count += 20
                torch.cuda.synchronize()
            e1.record()
            e1.synchronize()
            out[name] = {"burst_tflops": flop / (best * 1e-3) / 1e12,
                         "sustained_tflops": flop * count / (e0.elapsed_time(e1) * 1e-3) / 1e12}
    clocks = clk.summary()
    line = {"peaks": out, "clocks": clocks, "n": n}
    text = (
        "# Dense e4m3 matmul peak of this B200 (the denominator of the fp8 rooflines)\n\n"
        "Command (one GPU, no profiler): `python bench.py --measure-peak`\n\n"
        f"8192^3 matmuls through torch (cuBLASLt): e4m3 x e4m3 -> bf16 with unit fp32 scales "
        f"(torch._scaled_mm) and bf16 x bf16 (torch.matmul); burst = best of {steps_burst} "
        f"single runs, sustained = back-to-back runs for {sustain_s:.0f} s under the power cap; "
        "CUDA events.\n\n"
        f"e4m3_tflops: {out['e4m3']['burst_tflops']:.1f}\n"
        f"e4m3_tflops_sustained: {out['e4m3']['sustained_tflops']:.1f}\n"
        f"bf16_tflops_same_run: {out['bf16']['burst_tflops']:.1f}\n"
        f"bf16_tflops_sustained_same_run: {out['bf16']['sustained_tflops']:.1f}\n"
        f"sm_mhz_median: {clocks.get('sm_mhz')}\n"
        f"sm_max_mhz: {clocks.get('sm_max_mhz')}\n"
        f"throttle_reasons: {', '.join(clocks.get('reasons') or []) or 'none'}\n"
    )
    with open(E4M3_PEAK_FILE, "w") as f:
        f.write(text)
    print(json.dumps(line), flush=True)


def kernel_source_hash() -> str:
    """Hash of what the grouped-GEMM kernels are compiled from: their sources
    (the 128 x 256 kernel and the per-group-scale one), the shared tile
    schedule, the PTX helpers, the common helpers and their argument struct
    (the rest of the launcher header does not change the kernels)."""
    csrc = os.path.join(ROOT, "top_routing_grouped_gemv_b200", "csrc")
    h = hashlib.sha256()
    for name in ("gemm_tc.cu", "gemm_gs.cu", "grouped_tiles.cuh", "tc_ptx.cuh", "common.cuh"):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    with open(os.path.join(csrc, "kernels.h")) as f:
        hdr = f.read()
    m = re.search(r"struct TcGemmArgs \{.*?\n\};", hdr, re.S)
    h.update((m.group(0) if m else hdr).encode())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str, kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, if
    it was taken on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_sha = re.search(r"kernel_source_sha256_16:\s*([0-9a-f]+)", text)
    m_b = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not m_sha or not m_b or m_sha.group(1) != kernel_source_hash():
        return None
    return float(m_b.group(1))


class ClockSampler:
    """NVML sampling of SM clock and throttle reasons on this process's GPU."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples, self.reasons, self.ok = [], 0, False
        self.period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            uuid = None
            try:
                import torch
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            except Exception:
                pass
            h = None
            if uuid:
                for i in range(pynvml.nvmlDeviceGetCount()):
                    hh = pynvml.nvmlDeviceGetHandleByIndex(i)
                    u = pynvml.nvmlDeviceGetUUID(hh)
                    u = u.decode() if isinstance(u, bytes) else u
                    if u.replace("GPU-", "") == uuid.replace("GPU-", ""):
                        h = hh
            self.h = h or pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report that, keep going
            self.err = str(e)

    def _run(self):
        nv = self.nv
        while not self.stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.stop = threading.Event()
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self.stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.err}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


def max_over_ranks(value: float, dist=None, device: str = "cuda") -> float:
    """The largest `value` over all ranks (timings of replicas are reported
    as the slowest rank's); identity without a process group."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(tokens_per_rank_step: int, steps: int, world: int, max_ms: float) -> float:
    """Whole-job tokens/s of `world` independent replicas, each processing
    tokens_per_rank_step tokens per step, over the slowest rank's time."""
    return world * tokens_per_rank_step * steps / (max_ms / 1e3)


def R_rows(cfg) -> int:
    """Routed rows of a layer (tokens x experts per token)."""
    return cfg.N * cfg.K


def gemm_flops(cfg, rows: int):
    """Algorithmic FLOPs of the grouped FFN over the actual routed rows."""
    if cfg.act == "swiglu":
        return 2.0 * rows * cfg.d * 2 * cfg.F, 2.0 * rows * cfg.F * cfg.d
    if cfg.act == "relu":
        return 2.0 * rows * cfg.d * cfg.F, 2.0 * rows * cfg.F * cfg.d
    return 2.0 * rows * cfg.d * cfg.F, 0.0


def oracle_tokens(inp, tok):
    """The oracle's layer on tokens `tok`: the whole forward, or for the MX
    layer its K rows per token through the MX experts (pure unpermute)."""
    import numpy as np
    import oracle
    cfg = inp.cfg
    if cfg.quant in ("mx", "group", "block"):
        rows = np.repeat(np.asarray(tok), cfg.K)
        row_e = inp.ids.numpy()[tok].reshape(-1).astype(np.int32)
        if cfg.quant == "mx":
            return oracle.expert_rows_mx(row_e, inp.x.numpy()[rows], inp.x_sf.numpy()[rows],
                                         inp.w1, inp.w_sf)
        ws = inp.w_gs.numpy().astype(np.float64)
        if cfg.quant == "block":
            ws = oracle.block_to_group_scales(ws, cfg.F)
        return oracle.expert_rows_kscaled(row_e, inp.x.numpy()[rows], oracle.E4M3, inp.w1,
                                          oracle.E4M3, ws,
                                          x_group_scales=inp.x_gs.numpy()[rows])
    gm = 0 if cfg.routing == "given" else 1   # given routing: the pure unpermute
    return oracle.forward_tokens(inp, tok, gates_mode=gm)


def oracle_sample_tokens(cfg, inp, target_s: float, max_tokens: int | None = None):
    """Time the oracle's whole-layer forward on a token sample sized to take
    about target_s seconds; returns (tokens, seconds, threads)."""
    import numpy as np
    import oracle
    threads = oracle.num_threads()
    n = max(1, threads)
    t0 = time.perf_counter()
    oracle_tokens(inp, np.arange(n))
    dt = time.perf_counter() - t0
    n2 = int(min(max_tokens or cfg.N, max(n, n * target_s / max(dt, 1e-6))))
    n2 = max(threads, n2 // threads * threads) if n2 >= threads else n2
    rng = np.random.default_rng(17)
    tok = np.sort(rng.choice(cfg.N, size=min(n2, cfg.N), replace=False))
    t0 = time.perf_counter()
    oracle_tokens(inp, tok)
    return len(tok), time.perf_counter() - t0, threads


def run_reference(args, rank: int):
    import numpy as np
    import oracle
    import synth
    cfg = synth.CONFIGS[args.workload]
    if rank != 0:
        return
    oracle.build()
    inp = synth.make_inputs(cfg)
    threads = oracle.num_threads()
    per = max(1, threads)
    rng = np.random.default_rng(23)
    for _ in range(args.warmup):
        oracle_tokens(inp, rng.choice(cfg.N, size=per, replace=False))
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_tokens(inp, rng.choice(cfg.N, size=per, replace=False))
    dt = time.perf_counter() - t0
    value = per * args.steps / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": cfg.name, "N": cfg.N, "d": cfg.d, "E": cfg.E, "K": cfg.K,
                   "F": cfg.F, "act": cfg.act, "parallelism": "host cores"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": f"{per} random tokens of the {cfg.N}-token batch per step "
                                   "(route, K experts, combine), fp64"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, rank)
        return
    if args.measure_peak:
        if rank == 0:
            measure_peak()
        return

    import numpy as np
    import torch
    import synth
    import top_routing_grouped_gemv_b200 as moe

    assert torch.cuda.is_available(), "bench needs a CUDA device"
    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    moe.build()
    moe.load()

    cfg = synth.CONFIGS[args.workload]
    inp = synth.make_inputs(cfg)
    w = {"w1": inp.w1.cuda(), "w_scale": inp.w_scale}
    gkey = "w_block_scales" if cfg.quant == "block" else "w_group_scales"
    for k, t in (("w3", inp.w3), ("w2", inp.w2), ("w_r", inp.w_r), ("bias", inp.bias),
                 ("w_mx_scales", inp.w_sf), (gkey, inp.w_gs)):
        if t is not None:
            w[k] = t.cuda()
    plan = moe.Plan(cfg.N, cfg.d, cfg.E, cfg.K, cfg.F, cfg.dtype, cfg.act, w)
    ws = plan.new_workspace()
    x = inp.x.cuda()
    ydt = torch.float32 if cfg.dtype == "f32" else torch.bfloat16
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    given = cfg.routing == "given"
    mx = cfg.quant == "mx"
    gsq = cfg.quant in ("group", "block")
    shared = cfg.shared is not None
    ysh = xsf = None
    if given and gsq:
        # group / block-scaled grouped-matmul layer: the caller's routing and
        # per-token-and-group activation scales, unpermute in the GEMM's stores
        ids = inp.ids.cuda()
        xsf = inp.x_gs.cuda()
        y = torch.empty(cfg.N * cfg.K, cfg.d_out, dtype=ydt, device="cuda")

        def step():
            plan.forward_routed_group_scales(x, ids, None, y, ws, x_group_scales=xsf)
    elif given and mx:
        # MX grouped-matmul layer: the caller's routing and block scales, the
        # pure unpermute done by the GEMM's stores
        ids = inp.ids.cuda()
        xsf = inp.x_sf.cuda()
        y = torch.empty(cfg.N * cfg.K, cfg.d_out, dtype=ydt, device="cuda")

        def step():
            plan.forward_routed_mx(x, xsf, ids, None, y, ws)
    elif given:
        # fp8 grouped-matmul layer: the caller's routing, the pure unpermute
        # done by the GEMM's stores, and the shared expert on a forked stream
        ids = inp.ids.cuda()
        y = torch.empty(cfg.N * cfg.K, cfg.d_out, dtype=ydt, device="cuda")
        N2 = cfg.shared[1]
        wsh = inp.w_sh.cuda()
        ysh = torch.empty(cfg.N, N2, dtype=torch.bfloat16, device="cuda")

        def step():
            plan.forward_routed_shared(x, ids, None, y, wsh, inp.w_sh_scale, ysh, ws,
                                       x_scale=inp.x_scale)
    else:
        y = torch.empty(cfg.N, cfg.d_out, dtype=ydt, device="cuda")

        def step():
            plan.forward(x, y, ws)

    # warm-up
    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    assert plan.read_device_status(ws) == 0, "device status after warm-up"
    launches_per_step = plan.last_launch_count() + (1 if shared else 0)  # + the shared matmul

    # timed region: K steps back to back (the host runs ahead of the GPU),
    # CUDA events around every step on the launching stream
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        wall0 = time.perf_counter()
        for i in range(args.steps):
            flush.zero_()
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        torch.cuda.synchronize()
        wall = time.perf_counter() - wall0
        # per-kernel durations: the same loop with the library recording
        # events between its kernels.  Each iteration waits for its events, so
        # the host starts every step from idle: a GPU sleep after the L2 flush
        # (about 0.5 ms) gives it the head start it has in the timed loop, so
        # every launch is queued before the GPU reaches it and no host launch
        # delay lands inside a kernel's span (the first kernel's included)
        plan.profile(True)
        per_kernel: dict[str, list[float]] = {}
        for i in range(min(args.steps, 100)):
            flush.zero_()
            torch.cuda._sleep(1_000_000)
            step()
            for name, ms in plan.profile_read():
                per_kernel.setdefault(name, []).append(ms)
        plan.profile(False)
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = max_over_ranks(sum(step_ms), dist)
    assert plan.read_device_status(ws) == 0, "device status after timing"
    value = replica_throughput(cfg.N, args.steps, world, total_ms)

    # end to end through the host-buffer entry point: each step copies its
    # batch in from pinned host memory and its result back out
    # (moe_forward_host_async: the copies of one step overlap the compute of
    # its neighbours, as in a serving loop); device events from before the
    # first H2D to after the last D2H
    e2e = None
    if not args.no_e2e and given:
        # fp8 layers: each step copies its x (and MX scales) and routing in
        # from pinned host memory, runs the routed layer (and the shared
        # expert), and copies the results back (no host-buffer entry point
        # for these layers: the copies are queued on the compute stream)
        ins = [(x, inp.x.clone().pin_memory()), (ids, inp.ids.clone().pin_memory())]
        if mx or gsq:
            ins.append((xsf, (inp.x_sf if mx else inp.x_gs).clone().pin_memory()))
        outs = [(y, torch.empty(tuple(y.shape), dtype=y.dtype).pin_memory())]
        if shared:
            outs.append((ysh, torch.empty(tuple(ysh.shape), dtype=ysh.dtype).pin_memory()))

        def e2e_step():
            for dev, host in ins:
                dev.copy_(host, non_blocking=True)
            step()
            for dev, host in outs:
                host.copy_(dev, non_blocking=True)

        for _ in range(min(args.warmup, 3)):
            e2e_step()
        torch.cuda.synchronize()
        n_e2e = max(1, args.steps)
        if dist:
            dist.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        b.record(stream)
        b.synchronize()
        e_ms = max_over_ranks(a.elapsed_time(b), dist)
        assert plan.read_device_status(ws) == 0, "device status after the host-buffer loop"
        e2e = {"value": replica_throughput(cfg.N, n_e2e, world, e_ms), "unit": "tokens/s",
               "h2d_bytes_per_step": sum(h.numel() * h.element_size() for _, h in ins),
               "d2h_bytes_per_step": sum(h.numel() * h.element_size() for _, h in outs),
               "steps": n_e2e,
               "api": ("moe_forward_routed_mx" if mx else "moe_forward_routed_group_scales" if gsq
                       else "moe_forward_routed_shared")
                      + " with pinned host copies on the same stream"}
    elif not args.no_e2e:
        xh = [inp.x.clone().pin_memory() for _ in range(2)]
        yh = [torch.empty(cfg.N, cfg.d_out, dtype=ydt).pin_memory() for _ in range(2)]
        for i in range(min(args.warmup, 3)):
            plan.forward_host_async(xh[i % 2], yh[i % 2], ws)
        plan.host_join()
        torch.cuda.synchronize()
        n_e2e = max(1, args.steps)
        if dist:
            dist.barrier()
        # no L2 flush in this loop: every step's x arrives fresh from the host
        # and the expert weights (> L2) are re-read each step anyway
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in range(n_e2e):
            plan.forward_host_async(xh[i % 2], yh[i % 2], ws)
        plan.host_join()
        b.record(stream)
        b.synchronize()
        e_ms = max_over_ranks(a.elapsed_time(b), dist)
        assert plan.read_device_status(ws) == 0, "device status after the host-buffer loop"
        e2e = {"value": replica_throughput(cfg.N, n_e2e, world, e_ms), "unit": "tokens/s",
               "h2d_bytes_per_step": xh[0].numel() * xh[0].element_size(),
               "d2h_bytes_per_step": yh[0].numel() * yh[0].element_size(), "steps": n_e2e,
               "api": "moe_forward_host_async (pinned host buffers, copies overlap neighbouring "
                      "steps' compute)"}

    # roofline of the dominant kernel
    peaks, peak_src = load_peaks()
    R = cfg.N * cfg.K
    f1, f2 = gemm_flops(cfg, R)
    k1 = "ffn1_swiglu_tc" if cfg.act == "swiglu" else (
        ("gmm_mx_tc" if mx else f"gmm_{cfg.quant}_tc" if gsq else "gmm_tc")
        if cfg.act == "none" else "ffn1_simt_f32")
    stage_us = {k: 1e3 * statistics.mean(v) for k, v in per_kernel.items()}
    if k1 not in stage_us and k1 + "_gather" in stage_us:
        k1 += "_gather"   # decode-shaped batches: the gate/up GEMM gathers its rows from x
    # decode-shaped layers (a few rows per expert) stream their weights: the
    # gate/up GEMM's bound is HBM, not the tensor pipe
    decode = cfg.dtype == "bf16" and cfg.act == "swiglu" and R_rows(cfg) <= 16 * cfg.E
    # the sustained (power-capped) peak applies to a kernel timed inside a long
    # loop or while the power cap throttles the clock; the burst one otherwise
    clk_summary = clk.summary()
    sustained = wall > 2.0 or "sw_power_cap" in clk_summary.get("reasons", [])
    peak = peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"]
    peak_desc = f"{peak_src} bf16 {'sustained' if sustained else 'burst'}"
    if cfg.dtype == "e4m3":
        p8 = load_e4m3_peak()
        if p8 is not None:   # the measured dense e4m3 matmul peak of this machine's B200s
            peak = p8["e4m3_tflops_sustained" if sustained else "e4m3_tflops"]
            peak_desc = (f"measured e4m3 {'sustained' if sustained else 'burst'} "
                         f"({os.path.relpath(E4M3_PEAK_FILE, ROOT)})")
        else:                # no measurement: 2x bf16, the nominal ratio
            peak *= 2.0
            peak_desc += " x 2 (e4m3 nominal ratio)"
    t1 = stage_us.get(k1, float("nan")) * 1e-6
    traffic = profiled_traffic(cfg.name, k1)
    if decode:
        # every expert's gate and up weights (R >= 4E: all experts are routed
        # to, but for a vanishing chance), the routed rows in, h out
        bytes1 = cfg.E * 2 * cfg.F * cfg.d * 2 + R * cfg.d * 2 + R * cfg.F * 2
        achieved = bytes1 / t1 / 1e9
        roofline = {"bound": "hbm", "kernel": k1, "achieved": achieved, "peak": peaks["hbm_gbs"],
                    "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
                    "peak_source": f"{peak_src} HBM copy bandwidth",
                    "algorithmic_bytes_per_launch": bytes1}
    else:
        achieved = f1 / t1 / 1e12
        roofline = {"bound": "tensor", "kernel": k1, "achieved": achieved, "peak": peak,
                    "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                    "peak_source": peak_desc,
                    "algorithmic_flop_per_launch": f1}
    ffn_keys = [k for k in stage_us if k.startswith("ffn") or k.startswith("gmm")]
    ffn_s = sum(stage_us[k] for k in ffn_keys) * 1e-6
    gemm = {"tflops": (f1 + f2) / ffn_s / 1e12, "frac_of_peak": (f1 + f2) / ffn_s / 1e12 / peak,
            "flop_per_step": f1 + f2}

    elem = {"f32": 4, "bf16": 2, "e4m3": 1}[cfg.dtype]
    mats = {"swiglu": 3, "relu": 2, "none": 1}[cfg.act]
    weight_mb = cfg.E * cfg.F * cfg.d * mats * elem / 1e6

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        n_tok, secs, threads = oracle_sample_tokens(cfg, inp, args.cpu_seconds)
        cpu = {"value": n_tok / secs, "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "sample": f"{n_tok} random tokens of the {cfg.N}-token batch (route, K experts, "
                         f"combine; fp64), {secs:.1f} s"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": cfg.dtype, "data": "synthetic",
            "config": {"workload": cfg.name, "N": cfg.N, "d": cfg.d, "E": cfg.E, "K": cfg.K,
                       "F": cfg.F, "act": cfg.act,
                       "router": ("given (top-K of seeded iid logits), OCP MXFP8 block scales "
                                  "(E8M0 per 32 elements)" if mx else
                                  f"given (top-K of seeded iid logits), fp32 {cfg.quant} scales "
                                  "(128-element groups of K)" if gsq else
                                  "given (top-K of seeded iid logits), shared expert "
                                  f"{cfg.shared[0]}x{cfg.shared[1]} on a forked stream")
                                 if given else "fp32",
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": "value: flushed (256 MiB write) before every step; e2e: inputs "
                             f"larger than L2 ({weight_mb:.0f} MB of expert weights), no flush",
                       "inputs": "seeded synthetic, resident in HBM"},
            "roofline": roofline, "gemm": gemm,
            "stages_us": {k: round(v, 2) for k, v in stage_us.items()},
            "cpu_baseline": cpu, "clocks": clk_summary, "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps,
        }
        print(json.dumps(line), flush=True)
    del plan
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
