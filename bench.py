"""Benchmark: SVDQuant W4A4 NVFP4 linear layer on B200.

One step = one ``svdq_w4a4_linear`` call (activation smoothing + NVFP4
quantize + low-rank down-projection, then the block-scaled FP4 GEMM with the
low-rank up-projection and bias) on the DiT MLP up-projection workload:
x bf16 [4096, 3072] -> y bf16 [4096, 12288], rank 32.  TFLOPS = 2 M N K / t
(the low-rank FLOPs are not counted).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 is launched with torchrun: every rank runs its own replica of the layer
on its own batch (tokens are independent; no collective on the data path),
time is the max over ranks, value = FLOPs of all ranks / that time.

``--impl reference`` times the CPU oracle (the plain numpy restatement in
oracle/) on a bounded sample of rows of the same workload.
Prints one JSON line (rank 0).
"""
import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "SVDQ W4A4 linear TFLOPS at M=4096,K=3072,N=12288 NVFP4; % of B200 FP4 peak"
WORKLOAD = "mlp_up"
FP4_SPEC_DENSE_TFLOPS = 9000.0      # NVIDIA B200 dense FP4 (18 PF is with 2:4 sparsity)
FP4_PER_BF16 = 4.0                  # nominal dense FP4 : BF16 throughput ratio
L2_BYTES = 126 * 2 ** 20

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one
# gemm_nvfp4_pair launch (the S2 kernel of this workload) from the ncu
# capture summarised in profiles/gemm_nvfp4_pair_mlp_up.md, keyed by the
# SHA-256 of the kernel sources it was taken from: once a source changes the
# figure no longer applies and the bench reports null.
GEMM_TRAFFIC = {
    "bytes": 30464768 + 51351808,
    "sources": {
        "bit_w4a4_diffusion_b200/csrc/gemm_nvfp4_pair.cu":
            "970105a4508e7e73ae94d34360d31df5931e56a058275e65edbaeac82990a07b",
        "bit_w4a4_diffusion_b200/csrc/epilogue.cuh":
            "c18b2678b535744d65b902ff8a6fbea589e0eb0a94e9e56de6a7c73e243609d9",
        "bit_w4a4_diffusion_b200/csrc/ptx.cuh":
            "d0ae4c9c0226adbd9ca9b7e6557ba21e131287ed65767747f8c97e2702b61e1e",
        "bit_w4a4_diffusion_b200/csrc/fused_quant.cuh":
            "f21ab85bdbe311d3d4165dcdeb812572d29a3cf396e766fb4835a66c8d267e4b",
        "bit_w4a4_diffusion_b200/csrc/svdq_internal.h":
            "3840be66fc764569e472c75b634ecd085965da9007331d9735442e2c86caae5a",
    },
}


def _measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def _gemm_traffic():
    import hashlib
    for rel, digest in GEMM_TRAFFIC["sources"].items():
        try:
            with open(os.path.join(ROOT, rel), "rb") as f:
                if hashlib.sha256(f.read()).hexdigest() != digest:
                    return None
        except OSError:
            return None
    return GEMM_TRAFFIC["bytes"]


# ------------------------------------------------------------------ ranks
# One process per GPU, each a replica on its own batch (tokens are
# independent rows; no data-path collective).  The only cross-rank steps are
# the barriers around the timed region and the max over ranks of its
# duration; `value` counts the tokens of all ranks.

def rank_barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def rank_max(v, world, device=None):
    """max over ranks of a per-rank duration (every rank gets it)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_rank_step, steps, world, max_ms):
    """TFLOP/s of the whole job: every rank's work over the slowest rank's time."""
    return world * flops_per_rank_step * steps / (max_ms * 1e-3) / 1e12


def _cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 0) for d in threadpool_info() if d.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def workload_config(M, K, N, world):
    """The `config` object of both arms' JSON lines (identical by construction)."""
    per_set = M * K * 2 + M * N * 2 + N * K // 2 + N * K // 16 + N * 128
    nsets = max(2, -(-2 * L2_BYTES // per_set))
    return {"workload": f"DiT MLP up-projection, svdq_w4a4_linear NVFP4 r32: x bf16 [{M},{K}] -> "
                        f"y bf16 [{M},{N}] (quantize + low-rank down-proj, FP4 GEMM + low-rank up-proj + bias)",
            "M": M, "K": K, "N": N, "rank": 32, "global_batch_tokens": M * world,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": f"rotating {nsets} weight/activation/output sets ({nsets * per_set / 2**20:.0f} MiB "
                  f"> 126 MiB L2)"}


# ------------------------------------------------------------------ oracle arm

def oracle_offline(inp, precision="nvfp4"):
    """The oracle's offline weight pack and weight dequantization (untimed)."""
    from oracle import svdq as O
    pw = O.pack_weights(precision, inp.W, inp.lam, inp.L1, inp.L2)
    return pw, O.dequantized_weight(precision, pw)


def oracle_step_fn(case, inp, rows_per_step, offline, precision="nvfp4"):
    """Per step: the oracle's activation quantization and fp64 layer output for
    `rows_per_step` rows (cycling through x)."""
    from oracle import svdq as O
    pw, deq_w = offline
    L1 = inp.L1.astype(np.float64)
    L2 = inp.L2.astype(np.float64)
    state = {"r0": 0}
    s_a = np.float32(inp.act_scale) if precision == "nvfp4" else None

    def step():
        r0 = state["r0"]
        rows = (np.arange(rows_per_step) + r0) % case.M
        state["r0"] = (r0 + rows_per_step) % case.M
        act = O.quantize_activations(precision, inp.x[rows], pw["inv_lam"], s_a)
        y = O.dequantized_act(precision, act) @ deq_w.T
        y += (act["x_hat"].astype(np.float64) @ L1) @ L2
        if inp.bias is not None:
            y += inp.bias[None, :]
        return y

    return step


def time_oracle(case, inp, steps, warmup, budget_s, precision="nvfp4"):
    """Returns (TFLOPS, seconds per step, rows per step)."""
    offline = oracle_offline(inp, precision)
    probe = oracle_step_fn(case, inp, min(32, case.M), offline, precision)
    probe()
    t0 = time.perf_counter()
    probe()
    t_row = (time.perf_counter() - t0) / min(32, case.M)
    rows = int(max(1, min(case.M, budget_s / max(steps + warmup, 1) / max(t_row, 1e-6))))
    fn = oracle_step_fn(case, inp, rows, offline, precision)
    for _ in range(warmup):
        fn()
    t0 = time.perf_counter()
    for _ in range(steps):
        fn()
    dt = (time.perf_counter() - t0) / steps
    return 2.0 * rows * case.N * case.K / dt / 1e12, dt, rows


def time_oracle_configs(budget_s):
    """The CPU oracle on every workload (a bounded sample of rows each, about
    `budget_s` seconds per config), plus the tiny layer on one thread: the
    per-config CPU baseline.  Host only."""
    import workloads as wl
    from oracle import awq as OA
    from oracle import calibrate as OC
    out = {}
    for name, prec in (("tiny", "nvfp4"), ("qkv", "nvfp4"), ("mlp_up", "nvfp4"), ("mlp_down", "nvfp4"),
                       ("int4_m4096", "int4")):
        case = wl.SVDQ_CASES[name]
        inp = wl.make_svdq_inputs(case, OC.calibrate)
        tf, dt, rows = time_oracle(case, inp, 2, 1, budget_s, prec)
        out[name] = {"precision": prec, "TFLOPS": round(tf, 6), "rows_timed": rows, "s_per_step": round(dt, 3)}
        if name == "tiny":
            try:
                from threadpoolctl import threadpool_limits
                with threadpool_limits(limits=1):
                    tf1, dt1, rows1 = time_oracle(case, inp, 2, 1, budget_s, prec)
                out["tiny_1_thread"] = {"precision": prec, "TFLOPS": round(tf1, 6), "rows_timed": rows1,
                                        "s_per_step": round(dt1, 3)}
            except ImportError:
                pass
    a = wl.make_awq_inputs(1)
    q, sc, z = OA.awq_quantize(a.W)
    OA.awq_linear(a.x, q, sc, z)
    t0 = time.perf_counter()
    reps = 3
    for _ in range(reps):
        OA.awq_linear(a.x, q, sc, z)
    dt = (time.perf_counter() - t0) / reps
    wbytes = a.N * a.K // 2 + a.N * a.K // 64 * 2 + a.N * a.K // 128
    out["awq_m1"] = {"GB/s": round(wbytes / dt / 1e9, 3), "s_per_call": round(dt, 4),
                     "note": "each timed call dequantizes W and multiplies in fp64"}
    out["cores"] = _cpu_threads()
    return out


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, index, period_s=0.005):
        self.samples, self.reasons, self.period = [], set(), period_s
        self.power_mw = []
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.power_mw.append(self.nv.nvmlDeviceGetPowerUsage(self.h))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._stop = threading.Event()
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        out = {"sm_mhz": float(statistics.median(self.samples)) if self.samples else None,
               "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons - {"gpu_idle"}),
               "samples": len(self.samples)}
        if self.power_mw:
            out["power_w_max"] = round(max(self.power_mw) / 1e3, 1)
        return out


# ------------------------------------------------------------------ GPU arm

def run_gpu(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import bit_w4a4_diffusion_b200 as B
    import workloads as wl

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    case = wl.SVDQ_CASES[WORKLOAD]
    inp = wl.make_svdq_inputs(case, B.svdq_calibrate)
    pk = B.svdq_pack_weights("nvfp4", inp.W_bits, inp.lam, inp.L1_bits, inp.L2_bits)
    s_a = float(inp.act_scale)
    M, N, K = case.M, case.N, case.K
    flops = 2.0 * M * N * K

    # Rotate over enough independent weight / activation / output sets that
    # a step's working set is never L2-resident from the previous use.
    per_set = M * K * 2 + M * N * 2 + N * K // 2 + N * K // 16 + N * 128
    nsets = max(2, -(-2 * L2_BYTES // per_set))
    sets = []
    x0 = B.bits_to_bf16(inp.x_bits, dev)
    bias = B.bits_to_bf16(inp.bias_bits, dev) if inp.bias_bits is not None else None
    for i in range(nsets):
        w = B.to_device(pk, dev)
        sets.append(dict(w=w, x=x0.clone(), y=torch.empty((M, N), dtype=torch.bfloat16, device=dev),
                         ws=torch.zeros(B.workspace_bytes("nvfp4", M, N, K), dtype=torch.uint8, device=dev),
                         codes=torch.empty((M, K // 2), dtype=torch.uint8, device=dev),
                         scales=torch.empty(B.act_scale_bytes("nvfp4", M, K), dtype=torch.uint8, device=dev),
                         lora=torch.empty((M, 64), dtype=torch.bfloat16, device=dev)))
    stream = torch.cuda.current_stream(dev)
    alpha = float(np.float32(np.float32(s_a) * np.float32(pk["weight_scale"][0])))

    def layer(i, st=None):
        s = sets[i % nsets]
        B.svdq_w4a4_linear("nvfp4", s["x"], s["w"], s_a, bias=bias, y=s["y"], workspace=s["ws"],
                           stream=st if st is not None else torch.cuda.current_stream(dev))

    def barrier():
        rank_barrier(world)

    def max_over_ranks(v):
        return rank_max(v, world, dev)

    # ---- timed region: K steps of the whole layer, replayed from a CUDA graph
    # of G consecutive steps (rotating the sets) so host launch cost is off the
    # critical path; a remainder is launched eagerly.
    for i in range(args.warmup):
        layer(i)
    torch.cuda.synchronize()
    G = nsets * max(1, 16 // nsets)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(G):
            layer(i)
    graph.replay()
    torch.cuda.synchronize()
    reps, rem = divmod(args.steps, G)
    sampler = ClockSampler(local_rank)
    barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with sampler:
        torch.cuda._sleep(20_000_000)          # let the host queue run ahead of the GPU
        e0.record(stream)
        for _ in range(reps):
            graph.replay()
        for i in range(rem):
            layer(i)
        e1.record(stream)
        torch.cuda.synchronize()
    barrier()
    t_ms = max_over_ranks(e0.elapsed_time(e1))
    ms_per_step = t_ms / args.steps
    value = whole_job_tflops(flops, args.steps, world, t_ms)

    # ---- sustained: the same graph replayed back to back for >= args.sustain_s
    # seconds (the power cap and clocks settle), timed the same way.
    sustained = None
    if args.sustain_s > 0:
        sreps = max(1, int(np.ceil(args.sustain_s * 1e3 / (ms_per_step * G))))
        ssampler = ClockSampler(local_rank)
        barrier()
        torch.cuda.synchronize()
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)
        with ssampler:
            torch.cuda._sleep(20_000_000)
            s0.record(stream)
            for _ in range(sreps):
                graph.replay()
            s1.record(stream)
            torch.cuda.synchronize()
        barrier()
        ts_ms = max_over_ranks(s0.elapsed_time(s1))
        us_step = ts_ms * 1e3 / (sreps * G)
        clk = ssampler.summary()
        sustained = {"seconds": round(ts_ms / 1e3, 3), "steps": sreps * G, "us_per_step": round(us_step, 2),
                     "value": round(whole_job_tflops(flops, sreps * G, world, ts_ms), 2), "clocks": clk}
        if clk.get("sm_mhz"):
            sustained["kcycles_per_step"] = round(us_step * clk["sm_mhz"] / 1e3, 2)

    # ---- per-kernel durations (events around each kernel, same rotation)
    nk = max(20, min(args.steps, 400))
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(nk)]
    torch.cuda._sleep(100_000_000)             # host enqueues all launches before the GPU reaches them
    for i in range(nk):
        s = sets[i % nsets]
        ev[i][0].record(stream)
        B.svdq_quantize_act("nvfp4", s["x"], s["w"]["inv_smooth"], s["w"]["lora_down"], s_a,
                            s["w"]["weight_scale_f"], out=(s["codes"], s["scales"], s["lora"]), stream=stream)
        ev[i][1].record(stream)
        B.svdq_w4a4_gemm("nvfp4", s["codes"], s["scales"], s["lora"], s["w"], alpha, bias=bias, y=s["y"],
                         stream=stream)
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    t_s1 = sum(e[0].elapsed_time(e[1]) for e in ev) / nk * 1e3    # us
    t_s2 = sum(e[1].elapsed_time(e[2]) for e in ev) / nk * 1e3

    # ---- end to end through the public API with host buffers: every step
    # copies its x in from pinned host memory and its y back out, pipelined
    # over three streams (copy in / compute / copy out, which use separate
    # copy engines), so that step i's output copy overlaps step i+1's input
    # copy and layer.  Buffer reuse across the rotating sets is ordered by
    # events.
    x_host = inp.x_bits.view(np.int16)
    hx = torch.from_numpy(x_host).view(torch.bfloat16).pin_memory()
    hys = [torch.empty((M, N), dtype=torch.bfloat16).pin_memory() for _ in range(nsets)]
    ke = max(20, min(50, args.steps // 10))
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_steps(n):
        done_layer, done_out = [None] * nsets, [None] * nsets
        last = None
        for i in range(n):
            k = i % nsets
            s = sets[k]
            with torch.cuda.stream(s_in):
                if done_layer[k] is not None:
                    s_in.wait_event(done_layer[k])      # layer i - nsets has read this x
                s["x"].copy_(hx, non_blocking=True)
                ev_in = torch.cuda.Event()
                ev_in.record(s_in)
            stream.wait_event(ev_in)
            if done_out[k] is not None:
                stream.wait_event(done_out[k])          # y of step i - nsets has left
            layer(i)
            done_layer[k] = torch.cuda.Event()
            done_layer[k].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(done_layer[k])
                hys[k].copy_(s["y"], non_blocking=True)
                done_out[k] = torch.cuda.Event()
                done_out[k].record(s_out)
            last = done_out[k]
        stream.wait_event(last)

    e2e_steps(2)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    f0 = torch.cuda.Event(enable_timing=True)
    f1 = torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    s_in.wait_stream(stream)
    e2e_steps(ke)
    f1.record(stream)
    torch.cuda.synchronize()
    barrier()
    te_ms = max_over_ranks(f0.elapsed_time(f1))
    e2e_value = whole_job_tflops(flops, ke, world, te_ms)

    peaks, peak_src = _measured_peaks()
    fp4_peak = peaks["bf16_tflops"] * FP4_PER_BF16
    fp4_peak_sus = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]) * FP4_PER_BF16
    fp4_meas = measure_fp4_peak(torch, dev) if args.fp4_peak else None
    s2_tflops = flops / (t_s2 * 1e-6) / 1e12

    per_gpu = value / world
    pct_burst = {"spec_dense_9pf": round(100 * per_gpu / FP4_SPEC_DENSE_TFLOPS, 2),
                 "bf16x4_nominal": round(100 * per_gpu / fp4_peak, 2)}
    if fp4_meas and fp4_meas.get("tflops"):
        pct_burst["measured_fp4"] = round(100 * per_gpu / fp4_meas["tflops"], 2)
    pct_all = {"burst": pct_burst}
    if sustained is not None:
        sv = sustained["value"] / world
        pct_sus = {"spec_dense_9pf": round(100 * sv / FP4_SPEC_DENSE_TFLOPS, 2),
                   "bf16x4_nominal_sustained": round(100 * sv / fp4_peak_sus, 2)}
        if fp4_meas and fp4_meas.get("tflops"):
            pct_sus["measured_fp4"] = round(100 * sv / fp4_meas["tflops"], 2)
        pct_all["sustained"] = pct_sus
    s1_bytes = M * K * 2 + M * K // 2 + M * K // 16 + M * 64 * 2 + K * 4 + 32 * K * 2
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4", "data": "synthetic",
        "config": workload_config(M, K, N, world),
        "pct_of_fp4_peak": pct_all,
        "roofline": {"kernel": "gemm_nvfp4_pair (S2)", "bound": "tensor", "achieved": round(s2_tflops, 1),
                     "peak": round(fp4_peak, 1), "unit": "TFLOP/s", "frac": round(s2_tflops / fp4_peak, 4),
                     "peak_source": f"{peak_src} bf16 burst {peaks['bf16_tflops']} x {FP4_PER_BF16} "
                                    f"(nominal fp4:bf16 dense ratio)",
                     "traffic": _gemm_traffic(), "traffic_unit": "bytes per launch (ncu dram read + write)"},
        "kernels": {"quantize_act_us": round(t_s1, 2), "gemm_nvfp4_us": round(t_s2, 2),
                    "quantize_act_gbs": round(s1_bytes / (t_s1 * 1e-6) / 1e9, 1),
                    "quantize_act_hbm_frac": round(s1_bytes / (t_s1 * 1e-6) / 1e9 / peaks["hbm_gbs"], 4)},
        "e2e": {"value": round(e2e_value, 2), "unit": "TFLOPS", "h2d_bytes_per_step": int(M * K * 2),
                "d2h_bytes_per_step": int(M * N * 2), "steps": ke,
                "pipelining": "copy in / layer / copy out on three streams, steps overlapped"},
        "gpu_launches": 2 * args.steps,
        "graph": f"{G} steps per CUDA graph, {reps} replays + {rem} eager",
        "clocks": sampler.summary(),
    }
    if sustained is not None:
        out["sustained"] = sustained
    if fp4_meas:
        out["fp4_measured"] = fp4_meas
    if not args.no_rows:
        out["rows"] = measure_rows(B, wl, dev, peaks)
    if rank == 0 and not args.no_cpu_baseline:
        tf, dt, rows = time_oracle(case, inp, steps=3, warmup=1, budget_s=args.cpu_budget)
        out["cpu_baseline"] = {"value": round(tf, 6), "unit": "TFLOPS", "cores": _cpu_threads(), "kind": "oracle",
                               "sample": f"{rows} of {M} rows per step, 3 steps (numpy fp64 oracle, weight "
                                         f"pack and dequantization offline)",
                               "s_per_step": round(dt, 3)}
    return out


def measure_fp4_peak(torch, dev, n=8192, iters=10):
    """The box's own dense FP4 rate, used only as a denominator: torch's
    block-scaled NVFP4 matmul (a cuBLAS kernel) at n x n x n on random E2M1
    codes with unit E4M3 scales, best of `iters` CUDA-event timings."""
    try:
        a = torch.randint(0, 256, (n, n // 2), dtype=torch.uint8, device=dev).view(torch.float4_e2m1fn_x2)
        b = torch.randint(0, 256, (n, n // 2), dtype=torch.uint8, device=dev).view(torch.float4_e2m1fn_x2)
        sa = torch.ones((n, n // 16), device=dev).to(torch.float8_e4m3fn)
        sb = torch.ones((n, n // 16), device=dev).to(torch.float8_e4m3fn)
        for _ in range(3):
            torch._scaled_mm(a, b.t(), sa, sb, out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        best = None
        for _ in range(iters):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch._scaled_mm(a, b.t(), sa, sb, out_dtype=torch.bfloat16)
            e1.record()
            torch.cuda.synchronize()
            t = e0.elapsed_time(e1)
            best = t if best is None else min(best, t)
        return {"tflops": round(2.0 * n ** 3 / (best * 1e-3) / 1e12, 1), "shape": f"{n}^3",
                "source": "torch._scaled_mm NVFP4 (cuBLAS), unit block scales, best of "
                          f"{iters} (denominator only)"}
    except Exception as e:  # the measurement is context; the bench line stands without it
        return {"tflops": None, "error": str(e).splitlines()[0][:200]}


def _event_time_us(torch, fns, iters):
    """Median device time (us) of fns[i % len(fns)]() over `iters` launches,
    enqueued behind a GPU sleep so host launch cost never shows."""
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(iters)]
    for i in range(3):
        fns[i % len(fns)]()
    torch.cuda.synchronize()
    torch.cuda._sleep(50_000_000)
    for i, (a, b) in enumerate(ev):
        a.record()
        fns[i % len(fns)]()
        b.record()
    torch.cuda.synchronize()
    return float(np.median([a.elapsed_time(b) * 1e3 for a, b in ev]))


def measure_rows(B, wl, dev, peaks):
    """The other hot-path rows at their workload sizes: AWQ W4A16 (HBM GB/s)
    and the INT4 W4A4 layer over the token sweep (TOPS).  Weight sets rotate
    so that no launch finds its weights in L2."""
    import torch
    rows = {}
    awq = {}
    for M in wl.AWQ_MS:
        a = wl.make_awq_inputs(M)
        pk = B.awq_pack_weights(a.W_bits)
        nset = 6  # 6 x 30.5 MB > 126 MB L2
        ws = [B.to_device(pk, dev) for _ in range(nset)]
        x = B.bits_to_bf16(a.x_bits, dev)
        ys = [torch.empty((M, a.N), dtype=torch.bfloat16, device=dev) for _ in range(nset)]
        fns = [lambda i=i: B.awq_w4a16_linear(x, ws[i], y=ys[i]) for i in range(nset)]
        t = _event_time_us(torch, fns, 60)
        byts = a.N * a.K // 2 + a.N * a.K // 64 * 2 + a.N * a.K // 128 + M * a.K * 2 + M * a.N * 2
        awq[f"M={M}"] = {"us": round(t, 2), "GB/s": round(byts / t / 1e3, 1),
                         "hbm_frac": round(byts / t / 1e3 / peaks["hbm_gbs"], 3)}
        del ws, ys
    rows["awq_w4a16 N=18432 K=3072"] = awq
    int4 = {}
    for M in (1024, 2048, 4096, 8192):
        c = wl.SVDQ_CASES[f"int4_m{M}"]
        inp = wl.make_svdq_inputs(c, B.svdq_calibrate)
        pk = B.svdq_pack_weights("int4", inp.W_bits, inp.lam, inp.L1_bits, inp.L2_bits)
        nset = 4
        ws = [B.to_device(pk, dev) for _ in range(nset)]
        x = B.bits_to_bf16(inp.x_bits, dev)
        ys = [torch.empty((M, c.N), dtype=torch.bfloat16, device=dev) for _ in range(nset)]
        wsp = torch.zeros(B.workspace_bytes("int4", M, c.N, c.K), dtype=torch.uint8, device=dev)
        fns = [lambda i=i: B.svdq_w4a4_linear("int4", x, ws[i], 1.0, y=ys[i], workspace=wsp) for i in range(nset)]
        t = _event_time_us(torch, fns, 40)
        # The same layer with the other two GEMM options (for comparison).
        alt = {}
        for opt in ("dq", "i8"):
            os.environ["SVDQ_INT4_LAYER_GEMM"] = opt
            try:
                alt[opt] = _event_time_us(torch, fns, 40)
            finally:
                del os.environ["SVDQ_INT4_LAYER_GEMM"]
        int4[f"M={M}"] = {"us": round(t, 2), "TOPS": round(2.0 * M * c.N * c.K / t / 1e6, 1),
                          "dq_in_gemm_us": round(alt["dq"], 2), "i8_gemm_us": round(alt["i8"], 2)}
        del ws, ys
    int4["what"] = ("svdq_w4a4_linear INT4: quantize, both operands written out in fp16 (one launch), CTA-pair "
                    "fp16 GEMM; dq_in_gemm_us: the GEMM building its fp16 operand tiles from the codes itself; "
                    "i8_gemm_us: the i8 kernel of svdq_w4a4_gemm")
    rows["svdq_w4a4 int4 K=N=3072"] = int4
    rows["hbm_read_reference"] = measure_read_reference(dev, peaks)
    rows["mlp_gelu"] = measure_mlp(B, wl, dev)
    rows["qkv_norm_rope"] = measure_qkv(B, wl, dev)
    rows["dit_block"] = {f"M={M}": measure_block(B, wl, dev, M) for M in (4096, 1024)}
    return rows


def measure_read_reference(dev, peaks):
    """What one launch of a plain streaming read costs at the sizes of the
    HBM-bound rows (S1 reads 25 MB, S4 30.5 MB): torch's sum over a bf16
    tensor (a library kernel, used only as this reference), rotating over
    buffers that together exceed L2, timed like the rows."""
    import torch
    out = {}
    for mib in (8, 32, 128):
        n = mib * 2 ** 20 // 2
        nset = max(2, -(-2 * L2_BYTES // (mib * 2 ** 20)))
        bufs = [torch.randn(n, device=dev).to(torch.bfloat16) for _ in range(nset)]
        acc = torch.empty((), dtype=torch.float32, device=dev)
        fns = [lambda i=i: torch.sum(bufs[i], dim=0, dtype=torch.float32, out=acc) for i in range(nset)]
        t = _event_time_us(torch, fns, 40)
        out[f"{mib} MiB"] = {"us": round(t, 2), "GB/s": round(mib * 2 ** 20 / t / 1e3, 1),
                             "hbm_frac": round(mib * 2 ** 20 / t / 1e3 / peaks["hbm_gbs"], 3)}
        del bufs
    out["what"] = "torch.sum over a bf16 tensor (reads only), rotating buffers > L2, one launch each"
    return out


def measure_qkv(B, wl, dev, heads=24):
    """The DiT QKV projection (4096 tokens, 3072 -> 9216) with RMSNorm and
    RoPE on its Q and K heads: fused in the GEMM's epilogue, against the
    layer followed by the same normalization and rotation as separate bf16
    torch operations (for comparison only).  Two rotating weight sets."""
    import torch
    c = wl.SVDQ_CASES["qkv"]
    M, K, N = c.M, c.K, c.N
    inp = wl.make_svdq_inputs(c, B.svdq_calibrate)
    pk = B.svdq_pack_weights("nvfp4", inp.W_bits, inp.lam, inp.L1_bits, inp.L2_bits)
    nset = 2
    ws_ = [B.to_device(pk, dev) for _ in range(nset)]
    gq, gk, cos_m, sin_m = wl.make_rope_norm_inputs(M, heads)
    gq, gk = torch.from_numpy(gq).to(dev), torch.from_numpy(gk).to(dev)
    cos = torch.from_numpy(np.ascontiguousarray(cos_m.T)).to(dev)      # pair-major [64, M]
    sin = torch.from_numpy(np.ascontiguousarray(sin_m.T)).to(dev)
    x = B.bits_to_bf16(inp.x_bits, dev)
    bias = B.bits_to_bf16(inp.bias_bits, dev)
    s_a = float(inp.act_scale)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    wsp = torch.zeros(B.workspace_bytes("nvfp4", M, N, K), dtype=torch.uint8, device=dev)
    hd = heads * 128

    gq16, gk16 = gq.to(torch.bfloat16), gk.to(torch.bfloat16)
    c16 = cos.t().reshape(M, 1, 64).to(torch.bfloat16)
    s16 = sin.t().reshape(M, 1, 64).to(torch.bfloat16)

    def torch_norm_rope(t, g):
        n = torch.nn.functional.rms_norm(t.view(M, heads, 128), (128,), g, eps=1e-6)
        a, b = n[..., 0::2], n[..., 1::2]
        return torch.stack((a * c16 - b * s16, a * s16 + b * c16), dim=-1).view(M, hd)

    def unfused(i):
        B.svdq_w4a4_linear("nvfp4", x, ws_[i], s_a, bias=bias, y=y, workspace=wsp)
        y[:, :hd] = torch_norm_rope(y[:, :hd], gq16)
        y[:, hd:2 * hd] = torch_norm_rope(y[:, hd:2 * hd], gk16)

    fused = [lambda i=i: B.svdq_w4a4_qkv_norm_rope_linear(x, ws_[i], s_a, heads, gq, gk, cos, sin, bias=bias, y=y,
                                                          workspace=wsp) for i in range(nset)]
    plain = [lambda i=i: B.svdq_w4a4_linear("nvfp4", x, ws_[i], s_a, bias=bias, y=y, workspace=wsp)
             for i in range(nset)]
    t_f = _event_time_us(torch, fused, 40)
    t_p = _event_time_us(torch, plain, 40)
    t_u = _event_time_us(torch, [lambda i=i: unfused(i) for i in range(nset)], 40)
    flop = 2.0 * M * N * K
    del ws_
    return {"workload": f"x [{M},{K}] -> [{M},{N}], {heads} heads of 128, NVFP4 r32, bias",
            "fused_us": round(t_f, 2), "fused_TFLOPS": round(flop / t_f / 1e6, 1),
            "unfused_us": round(t_u, 2), "speedup": round(t_u / t_f, 3),
            "layer_without_norm_rope_us": round(t_p, 2)}


def block_layers(B, wl, dev, M, calibrate=None):
    """The linear layers of one DiT block at M tokens, hidden 3072: the
    adaptive-norm modulation (awq_w4a16, 1 row -> 6 x 3072), the fused QKV
    projection with RMSNorm and RoPE on Q and K (3072 -> 9216, 24 heads),
    the attention output projection
    (3072 -> 3072) and the GELU MLP (3072 -> 12288 -> 3072).  Attention,
    norms and residual adds are not part of this library; each layer reads
    its own synthetic input.  `calibrate` produces each layer's smoothing,
    low-rank factors and activation scale (the library's svdq_calibrate by
    default).  Returns a function that enqueues the block (its `inputs`
    attribute holds the host inputs of every layer and the workspace), the
    dict of output tensors and the block's FLOP count."""
    import dataclasses
    import torch
    cal = calibrate if calibrate is not None else B.svdq_calibrate
    q = wl.make_svdq_inputs(wl.scaled_case(wl.SVDQ_CASES["qkv"], M=M), cal)
    o = wl.make_svdq_inputs(wl.scaled_case(wl.SVDQ_CASES["qkv"], M=M, N=3072, name="attn_out"), cal)
    iu = wl.make_svdq_inputs(dataclasses.replace(wl.scaled_case(wl.SVDQ_CASES["mlp_up"], M=M), bias_std=0.1), cal)
    idn = wl.make_svdq_inputs(dataclasses.replace(wl.scaled_case(wl.SVDQ_CASES["mlp_down"], M=M), bias_std=0.05),
                              cal)
    a = wl.make_awq_inputs(1)
    rope = wl.make_rope_norm_inputs(M, 24)
    rq = [torch.from_numpy(np.ascontiguousarray(t.T if t.ndim == 2 else t)).to(dev) for t in rope]
    wq, wo, wu, wd = (B.to_device(B.svdq_pack_weights("nvfp4", i.W_bits, i.lam, i.L1_bits, i.L2_bits), dev)
                      for i in (q, o, iu, idn))
    wa = B.to_device(B.awq_pack_weights(a.W_bits), dev)
    xs = {k: B.bits_to_bf16(v, dev) for k, v in (("q", q.x_bits), ("o", o.x_bits), ("u", iu.x_bits),
                                                    ("a", a.x_bits))}
    bq = B.bits_to_bf16(q.bias_bits, dev) if q.bias_bits is not None else None
    bo = B.bits_to_bf16(o.bias_bits, dev) if o.bias_bits is not None else None
    bu, bd = B.bits_to_bf16(iu.bias_bits, dev), B.bits_to_bf16(idn.bias_bits, dev)
    out = {"mod": torch.empty((1, a.N), dtype=torch.bfloat16, device=dev),
           "qkv": torch.empty((M, 9216), dtype=torch.bfloat16, device=dev),
           "attn_out": torch.empty((M, 3072), dtype=torch.bfloat16, device=dev),
           "mlp": torch.empty((M, 3072), dtype=torch.bfloat16, device=dev)}
    ws = torch.zeros(max(B.workspace_bytes("nvfp4", M, 9216, 3072), B.mlp_workspace_bytes(M, 3072, 12288)),
                     dtype=torch.uint8, device=dev)

    def run():
        B.awq_w4a16_linear(xs["a"], wa, y=out["mod"])
        B.svdq_w4a4_qkv_norm_rope_linear(xs["q"], wq, float(q.act_scale), 24, *rq, bias=bq, y=out["qkv"],
                                         workspace=ws)
        B.svdq_w4a4_linear("nvfp4", xs["o"], wo, float(o.act_scale), bias=bo, y=out["attn_out"], workspace=ws)
        B.svdq_w4a4_mlp_gelu(xs["u"], wu, float(iu.act_scale), wd, float(idn.act_scale), up_bias=bu,
                             down_bias=bd, y=out["mlp"], workspace=ws)
    run.inputs = {"qkv": q, "attn_out": o, "mlp_up": iu, "mlp_down": idn, "awq": a, "rope": rope, "heads": 24,
                  "workspace": ws}
    flop = 2.0 * M * 3072 * (9216 + 3072 + 2 * 12288) + 2.0 * 18432 * 3072
    return run, out, flop


def measure_block(B, wl, dev, M, blocks=20):
    """One DiT block's linear layers, `blocks` blocks back to back: eager
    (each layer call launches its kernels) against one CUDA graph per block,
    each with and without programmatic dependent launch (SVDQ_PDL=0)."""
    import torch
    run, out, flop = block_layers(B, wl, dev, M)
    res = {}
    for pdl in (True, False):
        if pdl:
            os.environ.pop("SVDQ_PDL", None)
        else:
            os.environ["SVDQ_PDL"] = "0"
        try:
            for _ in range(3):
                run()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda._sleep(50_000_000)  # let the host queue the eager launches ahead
            e0.record()
            for _ in range(blocks):
                run()
            e1.record()
            torch.cuda.synchronize()
            eager = e0.elapsed_time(e1) * 1e3 / blocks
            g = torch.cuda.CUDAGraph()
            s = torch.cuda.Stream()
            s.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(s):
                run()
                torch.cuda.synchronize()
                with torch.cuda.graph(g, stream=s):
                    run()
            torch.cuda.current_stream().wait_stream(s)
            for _ in range(3):
                g.replay()
            torch.cuda.synchronize()
            e0.record()
            for _ in range(blocks):
                g.replay()
            e1.record()
            torch.cuda.synchronize()
            graph = e0.elapsed_time(e1) * 1e3 / blocks
            del g
        finally:
            os.environ.pop("SVDQ_PDL", None)
        tag = "pdl" if pdl else "no_pdl"
        res[f"eager_{tag}_us"] = round(eager, 2)
        res[f"graph_{tag}_us"] = round(graph, 2)
    res["graph_pdl_TFLOPS"] = round(flop / res["graph_pdl_us"] / 1e6, 1)
    res["layers"] = ("awq_w4a16 1x3072->18432, qkv+RMSNorm+RoPE 3072->9216, attn_out 3072->3072, "
                     "GELU MLP 3072->12288->3072")
    return res


def mlp_inputs(B, wl, dev, nset):
    """The DiT MLP block x [4096, 3072] -> 12288 -> 3072 (up: the mlp_up
    workload with a bias; down: the mlp_down workload's weights and
    calibration), `nset` device copies of both layers' packed weights."""
    import dataclasses
    iu = wl.make_svdq_inputs(dataclasses.replace(wl.SVDQ_CASES["mlp_up"], bias_std=0.1), B.svdq_calibrate)
    idn = wl.make_svdq_inputs(dataclasses.replace(wl.SVDQ_CASES["mlp_down"], bias_std=0.05), B.svdq_calibrate)
    pk_u = B.svdq_pack_weights("nvfp4", iu.W_bits, iu.lam, iu.L1_bits, iu.L2_bits)
    pk_d = B.svdq_pack_weights("nvfp4", idn.W_bits, idn.lam, idn.L1_bits, idn.L2_bits)
    wus = [B.to_device(pk_u, dev) for _ in range(nset)]
    wds = [B.to_device(pk_d, dev) for _ in range(nset)]
    return iu, idn, pk_u, wus, wds


def run_mlp_calls(calls):
    """`calls` back-to-back fused MLP calls on the DiT MLP workload, no
    timing (the command that the MLP profiles are taken with)."""
    import torch
    import bit_w4a4_diffusion_b200 as B
    import workloads as wl
    dev = torch.device("cuda:0")
    iu, idn, pk_u, wus, wds = mlp_inputs(B, wl, dev, 1)
    M, K, N = iu.case.M, iu.case.K, iu.case.N
    x = B.bits_to_bf16(iu.x_bits, dev)
    b_u = B.bits_to_bf16(iu.bias_bits, dev)
    b_d = B.bits_to_bf16(idn.bias_bits, dev)
    y = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    ws = torch.zeros(B.mlp_workspace_bytes(M, K, N), dtype=torch.uint8, device=dev)
    for _ in range(calls):
        B.svdq_w4a4_mlp_gelu(x, wus[0], float(iu.act_scale), wds[0], float(idn.act_scale), up_bias=b_u,
                             down_bias=b_d, y=y, workspace=ws)
    torch.cuda.synchronize()
    print(json.dumps({"mlp_calls": calls, "workload": f"x [{M},{K}] -> {N} -> {K}"}), flush=True)


def run_profile_calls(row, calls):
    """`calls` back-to-back calls of one row's entry point at its workload
    size, untimed (the commands the per-row profiles are taken with):
    awq (M = 1, N = 18432, K = 3072, six rotating weight sets), int4 (the
    INT4 layer at M = 4096, K = N = 3072, four sets), qkv (the fused QKV
    projection with RMSNorm and RoPE, two sets), mlp (the fused DiT MLP),
    layer (the headline NVFP4 layer, M = 4096, K = 3072, N = 12288, four
    sets), cublas_fp4 (for comparison only: torch's block-scaled NVFP4 matmul,
    a cuBLAS kernel, on the same shape with random codes and unit scales,
    three weight sets; no low-rank branch, no bias)."""
    import torch
    import bit_w4a4_diffusion_b200 as B
    import workloads as wl
    if row == "mlp":
        return run_mlp_calls(calls)
    dev = torch.device("cuda:0")
    if row == "awq":
        a = wl.make_awq_inputs(1)
        pk = B.awq_pack_weights(a.W_bits)
        ws = [B.to_device(pk, dev) for _ in range(6)]
        x = B.bits_to_bf16(a.x_bits, dev)
        y = torch.empty((1, a.N), dtype=torch.bfloat16, device=dev)
        fns = [lambda i=i: B.awq_w4a16_linear(x, ws[i], y=y) for i in range(6)]
    elif row == "int4":
        c = wl.SVDQ_CASES["int4_m4096"]
        inp = wl.make_svdq_inputs(c, B.svdq_calibrate)
        pk = B.svdq_pack_weights("int4", inp.W_bits, inp.lam, inp.L1_bits, inp.L2_bits)
        ws = [B.to_device(pk, dev) for _ in range(4)]
        x = B.bits_to_bf16(inp.x_bits, dev)
        y = torch.empty((c.M, c.N), dtype=torch.bfloat16, device=dev)
        wsp = torch.zeros(B.workspace_bytes("int4", c.M, c.N, c.K), dtype=torch.uint8, device=dev)
        fns = [lambda i=i: B.svdq_w4a4_linear("int4", x, ws[i], 1.0, y=y, workspace=wsp) for i in range(4)]
    elif row == "cublas_fp4":
        M, K, N = 4096, 3072, 12288
        a = torch.randint(0, 256, (M, K // 2), dtype=torch.uint8, device=dev).view(torch.float4_e2m1fn_x2)
        bs = [torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, device=dev).view(torch.float4_e2m1fn_x2)
              for _ in range(3)]
        sa = torch.ones((M, K // 16), device=dev).to(torch.float8_e4m3fn)
        sb = torch.ones((N, K // 16), device=dev).to(torch.float8_e4m3fn)
        fns = [lambda i=i: torch._scaled_mm(a, bs[i].t(), sa, sb, out_dtype=torch.bfloat16) for i in range(3)]
    elif row == "layer":
        c = wl.SVDQ_CASES[WORKLOAD]
        inp = wl.make_svdq_inputs(c, B.svdq_calibrate)
        pk = B.svdq_pack_weights("nvfp4", inp.W_bits, inp.lam, inp.L1_bits, inp.L2_bits)
        ws = [B.to_device(pk, dev) for _ in range(4)]
        x = B.bits_to_bf16(inp.x_bits, dev)
        bias = B.bits_to_bf16(inp.bias_bits, dev) if inp.bias_bits is not None else None
        y = torch.empty((c.M, c.N), dtype=torch.bfloat16, device=dev)
        wsp = torch.zeros(B.workspace_bytes("nvfp4", c.M, c.N, c.K), dtype=torch.uint8, device=dev)
        fns = [lambda i=i: B.svdq_w4a4_linear("nvfp4", x, ws[i], float(inp.act_scale), bias=bias, y=y, workspace=wsp)
               for i in range(4)]
    elif row == "qkv":
        c = wl.SVDQ_CASES["qkv"]
        inp = wl.make_svdq_inputs(c, B.svdq_calibrate)
        pk = B.svdq_pack_weights("nvfp4", inp.W_bits, inp.lam, inp.L1_bits, inp.L2_bits)
        ws = [B.to_device(pk, dev) for _ in range(2)]
        gq, gk, cm, sm = wl.make_rope_norm_inputs(c.M, 24)
        t = [torch.from_numpy(np.ascontiguousarray(v)).to(dev) for v in (gq, gk, cm.T, sm.T)]
        x = B.bits_to_bf16(inp.x_bits, dev)
        bias = B.bits_to_bf16(inp.bias_bits, dev)
        y = torch.empty((c.M, c.N), dtype=torch.bfloat16, device=dev)
        wsp = torch.zeros(B.workspace_bytes("nvfp4", c.M, c.N, c.K), dtype=torch.uint8, device=dev)
        fns = [lambda i=i: B.svdq_w4a4_qkv_norm_rope_linear(x, ws[i], float(inp.act_scale), 24, *t, bias=bias, y=y,
                                                            workspace=wsp) for i in range(2)]
    else:
        raise SystemExit(f"unknown row {row!r}")
    for i in range(calls):
        fns[i % len(fns)]()
    torch.cuda.synchronize()
    print(json.dumps({"profile_row": row, "calls": calls}), flush=True)


def measure_mlp(B, wl, dev):
    """The DiT MLP block, fused (the GELU and the down layer's activation
    quantizer in the up GEMM's epilogue) and unfused (up layer -> bf16 y ->
    GELU -> down layer; the GELU there is torch's, for comparison only).  Two
    rotating weight sets."""
    import torch
    nset = 2
    iu, idn, pk_u, wus, wds = mlp_inputs(B, wl, dev, nset)
    M, K, N = iu.case.M, iu.case.K, iu.case.N
    x = B.bits_to_bf16(iu.x_bits, dev)
    b_u = B.bits_to_bf16(iu.bias_bits, dev)
    b_d = B.bits_to_bf16(idn.bias_bits, dev)
    s_u, s_d = float(iu.act_scale), float(idn.act_scale)
    y = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    ws = torch.zeros(B.mlp_workspace_bytes(M, K, N), dtype=torch.uint8, device=dev)
    fused = [lambda i=i: B.svdq_w4a4_mlp_gelu(x, wus[i], s_u, wds[i], s_d, up_bias=b_u, down_bias=b_d, y=y,
                                              workspace=ws) for i in range(nset)]
    y_up = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    ws_u = torch.zeros(B.workspace_bytes("nvfp4", M, N, K), dtype=torch.uint8, device=dev)
    ws_d = torch.zeros(B.workspace_bytes("nvfp4", M, K, N), dtype=torch.uint8, device=dev)

    def unfused(i):
        B.svdq_w4a4_linear("nvfp4", x, wus[i], s_u, bias=b_u, y=y_up, workspace=ws_u)
        g = torch.nn.functional.gelu(y_up)
        B.svdq_w4a4_linear("nvfp4", g, wds[i], s_d, bias=b_d, y=y, workspace=ws_d)

    t_f = _event_time_us(torch, fused, 40)
    t_u = _event_time_us(torch, [lambda i=i: unfused(i) for i in range(nset)], 40)
    # the up GEMM alone, plain epilogue vs GELU-MLP epilogue
    codes, scales, lora = B.svdq_quantize_act("nvfp4", x, wus[0]["inv_smooth"], wus[0]["lora_down"], s_u,
                                              wus[0]["weight_scale_f"])
    alpha = float(np.float32(np.float32(s_u) * np.float32(pk_u["weight_scale"][0])))
    hc = torch.empty((M, N // 2), dtype=torch.uint8, device=dev)
    hs = torch.empty(B.act_scale_bytes("nvfp4", M, N), dtype=torch.uint8, device=dev)
    hl = torch.empty((M, 64), dtype=torch.bfloat16, device=dev)
    work = torch.empty(B.gelu_quant_work_bytes(M), dtype=torch.uint8, device=dev)
    t_plain = _event_time_us(torch, [lambda i=i: B.svdq_w4a4_gemm("nvfp4", codes, scales, lora, wus[i], alpha,
                                                                  bias=b_u, y=y_up) for i in range(nset)], 40)
    t_gq = _event_time_us(torch, [lambda i=i: B.svdq_w4a4_gemm_gelu_quant(
        codes, scales, lora, wus[i], alpha, wds[i], s_d, bias=b_u, out=(hc, hs, hl), work=work)
        for i in range(nset)], 40)
    flop = 2.0 * 2.0 * M * N * K
    del wus, wds
    return {"workload": f"x [{M},{K}] -> {N} -> {K}, NVFP4 r32, bias, exact GELU",
            "fused_us": round(t_f, 2), "fused_TFLOPS": round(flop / t_f / 1e6, 1),
            "unfused_us": round(t_u, 2), "unfused_TFLOPS": round(flop / t_u / 1e6, 1),
            "speedup": round(t_u / t_f, 3),
            "up_gemm_plain_us": round(t_plain, 2), "up_gemm_gelu_quant_us": round(t_gq, 2)}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=20.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-configs", action="store_true",
                    help="time the CPU oracle on every workload (host only) and print one JSON line")
    ap.add_argument("--no-rows", action="store_true", help="skip the INT4 / AWQ / MLP row measurements")
    ap.add_argument("--mlp-calls", type=int, default=0,
                    help="only run this many fused DiT MLP calls (untimed; for profiling) and exit")
    ap.add_argument("--profile", choices=["awq", "int4", "qkv", "mlp", "layer", "cublas_fp4"], default=None,
                    help="only run --calls calls of one row's entry point (untimed; for profiling) and exit")
    ap.add_argument("--calls", type=int, default=5)
    ap.add_argument("--sustain-s", type=float, default=2.0,
                    help="seconds of back-to-back graph replays for the sustained figure (0: skip)")
    ap.add_argument("--no-fp4-peak", dest="fp4_peak", action="store_false",
                    help="skip the measured FP4 denominator (torch._scaled_mm at 8192^3)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.mlp_calls > 0:
        run_mlp_calls(args.mlp_calls)
        return
    if args.profile is not None:
        run_profile_calls(args.profile, args.calls)
        return
    if args.cpu_configs:
        print(json.dumps({"cpu_oracle_configs": time_oracle_configs(args.cpu_budget / 2)}), flush=True)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return
        import workloads as wl
        from oracle import calibrate as OC
        case = wl.SVDQ_CASES[WORKLOAD]
        inp = wl.make_svdq_inputs(case, OC.calibrate)
        budget = max(30.0, min(150.0, 1.0 * (args.steps + args.warmup)))
        tf, dt, rows = time_oracle(case, inp, args.steps, args.warmup, budget)
        cores = _cpu_threads()
        sample = f"{rows} of {case.M} rows per step (numpy fp64 oracle; weight pack and dequantization offline)"
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": round(tf, 6), "unit": "TFLOPS", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(case.M, case.K, case.N, args.gpus),
            "cpu_baseline": {"value": round(tf, 6), "unit": "TFLOPS", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(tf, 6), "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }), flush=True)
        return

    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    out = run_gpu(args, rank, world, local_rank)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
