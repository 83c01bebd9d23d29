#!/usr/bin/env python
"""Benchmark of the gated delta rule on B200: prefill tokens/s (with its
fraction of the bf16 tensor-core roofline) and decode state-update HBM GB/s.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one chunkwise prefill of the 4 x 4096-token, 16 q/k-head,
32 v-head, d = 128, C = 64 bf16 workload (zero initial state), inputs
resident in HBM.  The decode step of the 256-sequence, 16/32-head, d = 128
workload (fp32 state of 512 MiB updated in place) is timed in the same run
and reported under "decode".  With N > 1 (torchrun) every rank runs an
independent replica on its own GPU (the problems are independent; there is
no data-path collective): "scaling" is "weak" and the value is the tokens
of all ranks over the slowest rank's device time.

The two other prefill workloads are timed in the same run and reported
under "long" (65,536 tokens, 16/48 heads, initial states) and "varlen" (32
packed sequences of 128..8192 tokens): each with its own roofline, e2e and
CPU baseline.

--impl reference times the fp64 CPU oracle on the host cores instead (on
rank 0 only): every step runs the oracle over the whole 4 x 4096 workload
(all (sequence, head) units), with the same code that times the GPU arm's
CPU baseline.
"""
from __future__ import annotations

import argparse
import hashlib
import ctypes
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GDN prefill tokens/s (% of bf16 TC peak); decode state-update HBM GB/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# Useful chunk FLOPs per (token, v-head) at d = 128, C = 64 with 2 v-heads per
# q/k head: inter-chunk 6 d^2 + triangular intra-chunk 3 C d + shared Gram 2 C d / G.
USEFUL_FLOPS_PER_VHEAD_TOKEN = 6 * 128 * 128 + 3 * 64 * 128 + 2 * 64 * 128 // 2


def parse_args(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--decode-steps", type=int, default=512)
    p.add_argument("--workload", choices=["prefill", "long", "varlen"], default="prefill",
                   help="prefill: 4 x 4096 tokens (the headline line); long: 65,536 tokens, 48 v heads, "
                        "initial states; varlen: 32 packed sequences of 128..8192 tokens")
    p.add_argument("--only", choices=["all", "prefill", "decode"], default="all",
                   help="time only one of the two paths (used by profiling commands)")
    p.add_argument("--raw-inputs", action="store_true",
                   help="prefill on raw q/k and gate logits, normalised and gated inside the kernels")
    p.add_argument("--output-norm", action="store_true",
                   help="prefill with the output side (RMS norm, per-channel scale, SiLU gate) in the kernel")
    p.add_argument("--kda", action="store_true",
                   help="Kimi Delta Attention (one decay per key channel) instead of the gated delta rule: "
                        "CUDA-core prefill (ALU roofline) and decode (HBM roofline)")
    p.add_argument("--backward", action="store_true",
                   help="time the gradients (training) on the prefill workload instead of the forward "
                        "(CUDA-core kernel, fp32 ALU roofline)")
    p.add_argument("--conv", type=int, default=0,
                   help="time the input side's short causal convolution with SiLU (this width) over q, k and v "
                        "of the prefill workload instead of the mixer (HBM roofline)")
    p.add_argument("--mtp", type=int, default=0,
                   help="decode: verify K draft tokens per sequence in one pass (state after every token kept)")
    p.add_argument("--split", action="store_true",
                   help="prefill through the two-kernel tensor-core form (chunk factors for all chunks, then the "
                        "chunk loop) instead of the default single kernel")
    p.add_argument("--no-graph", action="store_true",
                   help="decode: launch each step instead of replaying the ring of steps as one CUDA graph")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-extra", action="store_true",
                   help="time only the headline prefill workload (not the long-context and varlen records)")
    p.add_argument("--cpu-seconds", type=float, default=10.0, help="target CPU time of the oracle sample")
    return p.parse_args(argv)


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_traffic(kernel: str):
    """DRAM bytes per launch from a committed ncu summary (keyed by
    "kernel/workload"), only if the kernel's source has not changed since the
    counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        entries = json.load(f)
    e = entries.get(kernel)
    if not e:
        return None
    # one source, or several (a path of more than one kernel): all unchanged
    sources = e.get("sources") or [{"source": e["source"], "source_sha256": e["source_sha256"]}]
    for item in sources:
        src = os.path.join(ROOT, item["source"])
        if not os.path.exists(src):
            return None
        with open(src, "rb") as f:
            if hashlib.sha256(f.read()).hexdigest() != item["source_sha256"]:
                return None
    return e["bytes_per_launch"]


class ClockSampler:
    """Polls SM clock and clock-event reasons through NVML while running."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80, "sync_boost": 0x10}

    def __init__(self, index: int, interval: float = 0.01):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.interval = interval
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:  # NVML unavailable: report no clocks rather than fail the bench
            self.nv = None

    def _sample(self):
        if self.nv is None:
            return
        try:
            self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            bits = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            for name, mask in self.REASONS.items():
                if bits & mask:
                    self.reasons.add(name)
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.interval)

    def __enter__(self):
        self._sample()
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def __exit__(self, *exc):
        self._sample()
        self._stop.set()
        self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def max_over_ranks(x: float, device, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_value(tokens_per_rank: int, ms_max: float, world: int) -> float:
    """Whole-job tokens/s: every rank processes its own replica of the workload;
    the slowest rank's device time bounds the job."""
    return world * tokens_per_rank / (ms_max / 1e3)


def barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def timed(fn, steps, stream):
    """Device time per call (ms) over ``steps`` calls, CUDA events on ``stream``."""
    import torch
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(steps):
        fn()
    end.record(stream)
    end.synchronize()
    return start.elapsed_time(end) / steps


def host_cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


class OracleRun:
    """The fp64 oracle over every (sequence, head) unit of a workload.

    The fp64 copies of the inputs are made once, outside any timing, and
    ``run()`` times one pass of the oracle over the whole workload on all host
    cores.  The GPU arm's CPU baseline and the reference arm both use this."""

    def __init__(self, w, inp):
        from oracle import oracle
        self.oracle = oracle
        f64 = lambda t: None if t is None else t.to(dtype=__import__("torch").float64).numpy()
        self.args = [f64(inp[n]) for n in ("q", "k", "v", "g", "beta")]
        self.s0 = f64(inp["initial_state"])
        self.cu = None if inp["cu_seqlens"] is None else inp["cu_seqlens"].numpy().astype("int64")
        self.threads = oracle.default_threads()
        self.w = w

    def run(self) -> float:
        t0 = time.perf_counter()
        self.oracle.recurrent(*self.args, initial_state=self.s0, cu_seqlens=self.cu, threads=self.threads)
        return time.perf_counter() - t0


def cpu_baseline(w, inp, target_s: float):
    """Whole-workload passes of the oracle until about ``target_s`` seconds
    (at least one); tokens/s = tokens / mean seconds per pass."""
    r = OracleRun(w, inp)
    times = [r.run()]
    while sum(times) < target_s and len(times) < 50:
        times.append(r.run())
    per = statistics.mean(times)
    return {"value": w.total_tokens / per, "unit": "tokens/s", "cores": r.threads, "kind": "oracle",
            "cpu_model": host_cpu_model(), "seconds_per_pass": per,
            "sample": f"the whole workload {w.name} (all {w.num_seqs * w.hv} (sequence, v-head) units), "
                      f"{len(times)} pass(es), not extrapolated"}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    from linear_attention_sequence_sm_b200 import inputs as I
    w = I.prefill_bf16()
    r = OracleRun(w, I.make_prefill_inputs(w))
    times = []
    for i in range(args.warmup + args.steps):
        dt = r.run()
        if i >= args.warmup:
            times.append(dt)
    step_s = statistics.mean(times)
    value = w.total_tokens / step_s
    sample = f"the whole workload {w.name} (all {w.num_seqs * w.hv} (sequence, v-head) units) every step"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded splitmix64)",
        "config": {"workload": w.name, "global_batch": w.batch, "seq_len": w.seq_len, "parallelism": "none (host cores)"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": r.threads, "kind": "oracle",
                         "cpu_model": host_cpu_model(), "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)
    return 0


def e2e_record(fwd, w, host, ws, flags, out_norm, steps, device, world, stream):
    """The prefill through the public call with host buffers: every step copies
    its inputs from pinned host memory and its outputs (o and the final
    states) back, inside the timed region."""
    import torch
    pin = {k: v.pin_memory() for k, v in host.items() if v is not None}
    dv0 = next(iter(v for k, v in pin.items() if k == "v"))
    o_shape, sf_shape = dv0.shape, (w.num_seqs, w.hv, w.d, w.d)
    h2d = sum(t.numel() * t.element_size() for t in pin.values())
    d2h = dv0.numel() * dv0.element_size() + w.num_seqs * w.hv * w.d * w.d * 4

    # Steps overlap across three streams, double-buffered: step i's inputs copy in while step i-1
    # computes and step i-2's results copy out (separate copy engines for the two directions).
    # Every step still copies its own inputs from pinned host memory and its own results back.
    s_in, s_out, comp = torch.cuda.Stream(device), torch.cuda.Stream(device), stream
    dbuf = [{k: torch.empty_like(v, device=device) for k, v in pin.items()} for _ in range(2)]
    obuf = [torch.empty(o_shape, dtype=dv0.dtype, device=device) for _ in range(2)]
    sbuf = [torch.empty(sf_shape, dtype=torch.float32, device=device) for _ in range(2)]
    ohost = [torch.empty(o_shape, dtype=dv0.dtype).pin_memory() for _ in range(2)]
    shost = [torch.empty(sf_shape, dtype=torch.float32).pin_memory() for _ in range(2)]
    ev_in, ev_comp, ev_out = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))
    for b in range(2):
        ev_comp[b].record(comp)
        ev_out[b].record(comp)
    it = [0]

    def e2e_step():
        b = it[0] % 2
        it[0] += 1
        x = dbuf[b]
        s_in.wait_event(ev_comp[b])  # the step that last read these input buffers has run
        with torch.cuda.stream(s_in):
            for k_ in x:
                x[k_].copy_(pin[k_], non_blocking=True)
        ev_in[b].record(s_in)
        comp.wait_event(ev_in[b])
        comp.wait_event(ev_out[b])  # the results last held in these output buffers have left
        with torch.cuda.stream(comp):
            fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], initial_state=x.get("initial_state"),
                cu_seqlens=x.get("cu_seqlens"), chunk_size=w.chunk, out=obuf[b], final_state=sbuf[b],
                workspace=ws, **flags, **out_norm(x))
        ev_comp[b].record(comp)
        s_out.wait_event(ev_comp[b])
        with torch.cuda.stream(s_out):
            ohost[b].copy_(obuf[b], non_blocking=True)
            shost[b].copy_(sbuf[b], non_blocking=True)
        ev_out[b].record(s_out)

    def e2e_timed(n):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(comp)
        s_in.wait_stream(comp)
        for _ in range(n):
            e2e_step()
        comp.wait_stream(s_out)
        e1.record(comp)
        e1.synchronize()
        return e0.elapsed_time(e1) / n

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize(device)
    barrier(world, device)
    e_ms = max_over_ranks(e2e_timed(max(3, min(steps, 20))), device, world)
    del dbuf, obuf, sbuf
    return {"value": world * w.total_tokens / (e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": e_ms,
            "overlap": "copy-in, compute and copy-out of consecutive steps on three streams, double-buffered"}


def prefill_record(args, w, host, device, world, rank, peaks, peak_src, e2e=True, cpu=True):
    """Times the prefill of workload ``w`` (inputs resident in HBM) and returns
    its record: ms per step (max over ranks), tokens/s of all ranks, the
    roofline of the dominant kernel, the e2e figure and the CPU baseline."""
    import torch
    from linear_attention_sequence_sm_b200 import gdn
    from linear_attention_sequence_sm_b200 import inputs as I
    flags = {"qk_l2norm": True, "gate_logits": True} if args.raw_inputs else {}
    suffix = ("_kda" if args.kda else "") + ("_split" if args.split else "") + \
        ("_raw_inputs" if args.raw_inputs else "") + \
        ("_output_norm" if args.output_norm else "") + ("_backward" if args.backward else "") + \
        (f"_conv{args.conv}" if args.conv else "")
    if args.kda:
        host["g"] = I.make_kda_gates(w)
    fwd = gdn.kda_forward if args.kda else gdn.chunk_forward
    out_weight = None
    if args.output_norm:
        host["out_gate"] = I.make_output_gate(w)
        out_weight = I.make_output_weight(w).to(device)
    dev = {k: (v.to(device) if v is not None else None) for k, v in host.items()}

    def out_norm(x):
        if not args.output_norm:
            return {}
        return {"output_norm": gdn.OutputNorm(weight=out_weight, gate=x["out_gate"], eps=1e-6, activation="silu")}

    o = torch.empty_like(dev["v"])
    sf = torch.empty((w.num_seqs, w.hv, w.d, w.d), dtype=torch.float32, device=device)
    split = {"split": True} if args.split and not args.kda else {}
    shape = gdn.make_shape(dev["q"], dev["v"], dev["cu_seqlens"], w.chunk, **split)
    ws = torch.empty(gdn.kda_workspace_size(shape) if args.kda else gdn.workspace_size(shape), dtype=torch.uint8,
                     device=device)
    stream = torch.cuda.current_stream(device)

    if args.backward:
        dev["dO"] = torch.from_numpy(I.normal(w.seed, "bwd_do", tuple(host["v"].shape))).to(dev["v"].dtype).to(device)
        bshape = gdn.make_shape(dev["q"], dev["v"], dev["cu_seqlens"], 32)
        nb = ctypes.c_size_t(0)
        gdn.LIB.gdn_chunk_backward_workspace_size(ctypes.byref(bshape), ctypes.byref(nb))
        bws = torch.empty(nb.value, dtype=torch.uint8, device=device)

    if args.conv:
        convs = []
        for n_, h_ in (("q", w.hk), ("k", w.hk), ("v", w.hv)):
            wt = torch.from_numpy(I.normal(w.seed, "conv_" + n_, (h_, w.d, args.conv), std=args.conv ** -0.5))
            convs.append((dev[n_], wt.float().to(device), torch.empty_like(dev[n_]),
                          torch.empty((w.num_seqs, h_, w.d, args.conv - 1), dtype=torch.float32, device=device)))

    def step():
        if args.conv:
            for x_, wt_, y_, so_ in convs:
                gdn.short_conv(x_, wt_, cu_seqlens=dev["cu_seqlens"], silu=True, out=y_, state_out=so_)
            return
        if args.backward:
            gdn.chunk_backward(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], dev["dO"],
                               initial_state=dev["initial_state"], cu_seqlens=dev["cu_seqlens"], workspace=bws)
            return
        fwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], initial_state=dev["initial_state"],
            cu_seqlens=dev["cu_seqlens"], out=o, final_state=sf, workspace=ws, chunk_size=w.chunk,
            **flags, **out_norm(dev), **split)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(device)
    barrier(world, device)
    torch.cuda.synchronize(device)
    n0 = gdn.launch_count()
    clocks = ClockSampler(device.index)
    with clocks:
        ms = timed(step, args.steps, stream)
        torch.cuda.synchronize(device)
    launches = gdn.launch_count() - n0
    barrier(world, device)
    ms_max = max_over_ranks(ms, device, world)
    tokens = w.total_tokens
    flops = useful_flops_per_vhead_token(w.hv // w.hk) * tokens * w.hv
    achieved_tflops = flops / (ms / 1e3) / 1e12
    # the default path: the single tensor-core kernel where the value heads come in
    # multiples of 4, else the two-kernel form (chunk factors, then the chunk loop)
    if not gdn_tc_active(gdn, dev, w):
        kernel_name = "gdn_chunk_simt"
    elif w.hv % 4 == 0 and not split:
        kernel_name = "gdn_chunk_tc"
    else:
        kernel_name = "gdn_chunk_inverse+gdn_chunk_chain"
    roofline = {"bound": "tensor", "achieved": achieved_tflops, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": achieved_tflops / peaks["bf16_tflops"],
                "traffic": kernel_traffic(f"{kernel_name}/{w.name}{suffix}"),
                "kernel": kernel_name,
                "peak_source": f"{peak_src} bf16 dense (burst)",
                "frac_vs_sustained": achieved_tflops / peaks["bf16_tflops_sustained"],
                "frac_vs_nominal_2250": achieved_tflops / 2250.0,
                "flops_per_launch": flops, "algorithmic_bytes_per_launch": prefill_bytes(w)}
    alu_peak = FP32_LANES_PER_SM * 2 * torch.cuda.get_device_properties(device).multi_processor_count * \
        (clocks.summary().get("sm_max_mhz") or 1965) * 1e6 / 1e12
    if args.backward and backward_tc_active(gdn, dev, w):
        # the tensor-core form: factors, chains, gradients (useful flops, each product once)
        bflops = backward_flops_per_vhead_token(w.d) * tokens * w.hv
        achieved = bflops / (ms / 1e3) / 1e12
        kname = "gdn_bwd_factor+gdn_bwd_chain+gdn_bwd_grad"
        roofline = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                    "frac": achieved / peaks["bf16_tflops"], "traffic": kernel_traffic(f"{kname}/{w.name}{suffix}"),
                    "kernel": kname, "peak_source": f"{peak_src} bf16 dense (burst)", "flops_per_launch": bflops}
    elif args.backward:
        # reverse mode of the token recurrence: 20 d^2 flops per (token, value head) (the forward
        # recomputed, 6 d^2, and the backward, 14 d^2); fp32 on CUDA cores
        bflops = 20 * w.d * w.d * tokens * w.hv
        achieved = bflops / (ms / 1e3) / 1e12
        roofline = {"bound": "alu", "achieved": achieved, "peak": alu_peak, "unit": "TFLOP/s",
                    "frac": achieved / alu_peak, "traffic": kernel_traffic(f"gdn_backward/{w.name}{suffix}"),
                    "kernel": "gdn_backward", "peak_source": "fp32 FMA lanes x 2 x max SM clock (derived)",
                    "flops_per_launch": bflops}
    if args.conv:
        # one read and one write of q, k and v, the filters, and the conv states written
        cbytes = conv_bytes(w, args.conv)
        cgbs = cbytes / (ms / 1e3) / 1e9
        roofline = {"bound": "hbm", "achieved": cgbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": cgbs / peaks["hbm_gbs"], "traffic": kernel_traffic(f"gdn_conv/{w.name}{suffix}"),
                    "kernel": "gdn_conv", "peak_source": f"{peak_src} HBM copy", "bytes_per_step": cbytes}
    if args.kda and gdn_tc_active(gdn, dev, w):
        # the chunkwise WY form on the tensor cores: the gated delta rule's useful flops
        # with the Gram per value head (G = 1: its decay differs per head)
        kflops = useful_flops_per_vhead_token(1, w.d, w.chunk) * tokens * w.hv
        achieved = kflops / (ms / 1e3) / 1e12
        roofline = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                    "frac": achieved / peaks["bf16_tflops"],
                    "traffic": kernel_traffic(f"gdn_kda_factor+gdn_kda_chain/{w.name}{suffix}"),
                    "kernel": "gdn_kda_factor+gdn_kda_chain", "peak_source": f"{peak_src} bf16 dense (burst)",
                    "flops_per_launch": kflops, "algorithmic_bytes_per_launch": prefill_bytes(w, kda=True)}
    elif args.kda:
        # token-order recurrence on CUDA cores: 7 d_v d_k fp32 flops per (token, value head)
        # (decay, two dot products, rank-1 write); peak = SMs x 128 fp32 lanes x 2 x max SM clock
        kflops = kda_flops_per_vhead_token(w.d) * tokens * w.hv
        achieved = kflops / (ms / 1e3) / 1e12
        roofline = {"bound": "alu", "achieved": achieved, "peak": alu_peak, "unit": "TFLOP/s",
                    "frac": achieved / alu_peak, "traffic": kernel_traffic(f"gdn_kda/{w.name}{suffix}"),
                    "kernel": "gdn_kda", "peak_source": "fp32 FMA lanes x 2 x max SM clock (derived)",
                    "flops_per_launch": kflops, "algorithmic_bytes_per_launch": prefill_bytes(w, kda=True)}
    rec = {"workload": w.name + suffix, "ms_per_step": ms_max, "tokens_per_s": aggregate_value(tokens, ms_max, world),
           "tokens": tokens, "roofline": roofline, "gpu_launches": launches, "clocks": clocks.summary(),
           "config": {"global_batch": w.num_seqs * world, "seq_len": w.seq_len, "heads_qk_v": [w.hk, w.hv],
                      "head_dim": w.d, "chunk": w.chunk, "initial_state": w.s0_std > 0,
                      "l2": f"inputs larger than L2 ({prefill_bytes(w) / 1e6:.0f} MB of mandatory traffic per step)"}}
    del o, sf
    if e2e and not args.no_e2e and not args.backward and not args.conv:
        rec["e2e"] = e2e_record(fwd, w, host, ws, flags, out_norm, args.steps, device, world, stream)
    # (raw inputs, the output side, KDA or gradients: the timed oracle covers the plain forward only)
    if cpu and rank == 0 and world == 1 and not args.no_cpu_baseline and not suffix:
        rec["cpu_baseline"] = cpu_baseline(w, host, args.cpu_seconds)
    del dev, ws
    torch.cuda.empty_cache()
    return rec


def decode_record(args, device, world, rank, peaks, peak_src):
    """Times the decode step of the 256-sequence workload (state in place)."""
    import torch
    from linear_attention_sequence_sm_b200 import gdn
    from linear_attention_sequence_sm_b200 import inputs as I
    dw = I.decode_bf16()
    stream = torch.cuda.current_stream(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(dw.seed + rank)
    state = torch.randn((dw.num_seqs, dw.hv, dw.d, dw.d), generator=gen, device=device) * dw.s0_std
    ring = [{k: v.to(device) for k, v in I.make_decode_inputs(dw, s).items()} for s in range(8)]
    od = torch.empty((dw.num_seqs, dw.hv, dw.d), dtype=torch.bfloat16, device=device)
    it = [0]
    if args.kda:
        for s_, x in enumerate(ring):
            x["g"] = I.make_kda_decode_gates(dw, s_).to(device)
    if args.mtp > 0:
        # K draft tokens per sequence: [N, K, H, d] inputs, one snapshot per token
        K = args.mtp
        ring = []
        for s_ in range(4):
            xs = [I.make_decode_inputs(dw, s_ * K + j) for j in range(K)]
            ring.append({n: torch.stack([x_[n] for x_ in xs], dim=1).to(device) for n in xs[0]})
        snaps = torch.empty((dw.num_seqs, K, dw.hv, dw.d, dw.d), dtype=torch.float32, device=device)
        od = torch.empty((dw.num_seqs, K, dw.hv, dw.d), dtype=torch.bfloat16, device=device)

    def dstep():
        x = ring[it[0] % len(ring)]
        it[0] += 1
        if args.mtp > 0:
            gdn.decode_multi(x["q"], x["k"], x["v"], x["g"], x["beta"], state, out=od, snapshots=snaps)
            return
        (gdn.kda_decode_step if args.kda else gdn.decode_step)(x["q"], x["k"], x["v"], x["g"], x["beta"], state,
                                                               out=od)

    for _ in range(max(3, args.warmup)):
        dstep()
    torch.cuda.synchronize(device)
    run, per_call = dstep, 1
    graph = None
    if not args.no_graph:
        # the ring of steps captured once and replayed: no host launch gaps between steps
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for _ in range(len(ring)):
                dstep()
        graph.replay()
        torch.cuda.synchronize(device)
        run, per_call = graph.replay, len(ring)
    barrier(world, device)
    n0 = gdn.launch_count()
    with ClockSampler(device.index) as dclocks:
        dms = timed(run, max(1, args.decode_steps // per_call), stream) / per_call
    # kernels replayed from the graph are not counted by the library's host-side counter
    launches = (gdn.launch_count() - n0) if graph is None else len(ring) * max(1, args.decode_steps // per_call)
    dms = max_over_ranks(dms, device, world)
    dbytes = decode_bytes(dw, kda=args.kda, mtp=args.mtp)
    dgbs = dbytes / (dms / 1e3) / 1e9
    rec = {"value": world * dgbs, "unit": "GB/s", "ms_per_step": dms, "steps": args.decode_steps,
           "tokens_per_s": world * dw.num_seqs * max(1, args.mtp) / (dms / 1e3),
           "workload": dw.name + (f"_mtp{args.mtp}" if args.mtp > 0 else ""),
           "roofline": {"bound": "hbm", "achieved": dgbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": dgbs / peaks["hbm_gbs"],
                        "traffic": kernel_traffic(f"gdn_decode/{dw.name}" + ("_kda" if args.kda else "")
                                                  + (f"_mtp{args.mtp}" if args.mtp > 0 else "")),
                        "kernel": "gdn_decode", "peak_source": f"{peak_src} HBM copy",
                        "frac_vs_nominal_8000": dgbs / 8000.0, "bytes_per_launch": dbytes},
           "gpu_launches": launches, "clocks": dclocks.summary(), "cuda_graph": not args.no_graph}
    del graph, state, ring
    torch.cuda.empty_cache()
    return rec


def run_ours(args):
    import torch
    rank, world, local_rank = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    from linear_attention_sequence_sm_b200 import inputs as I

    peaks, peak_src = load_peaks()
    makers = {"prefill": (I.prefill_bf16, 1002), "long": (I.long_bf16, 1003), "varlen": (I.varlen_bf16, 1005)}
    mk, seed = makers[args.workload]
    w = mk(seed=seed + rank)
    host = I.make_raw_prefill_inputs(w) if args.raw_inputs else I.make_prefill_inputs(w)

    head = None
    if args.only in ("all", "prefill"):
        head = prefill_record(args, w, host, device, world, rank, peaks, peak_src)
    del host
    # the other two prefill workloads, each with its own record (plain forward only)
    extra = {}
    plain = not (args.kda or args.raw_inputs or args.output_norm or args.backward or args.conv)
    if args.only == "all" and args.workload == "prefill" and plain and not args.no_extra:
        for name in ("long", "varlen"):
            mk2, seed2 = makers[name]
            w2 = mk2(seed=seed2 + rank)
            extra[name] = prefill_record(args, w2, I.make_prefill_inputs(w2), device, world, rank, peaks, peak_src)

    decode = None
    if args.only in ("all", "decode") and args.decode_steps > 0 and not args.conv:
        decode = decode_record(args, device, world, rank, peaks, peak_src)

    if rank == 0:
        ms_max = head["ms_per_step"] if head else float("nan")
        line = {
            "metric": METRIC, "value": head["tokens_per_s"] if head else None, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded splitmix64 / Box-Muller)",
            "config": dict({"workload": head["workload"] if head else w.name,
                            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
                           **(head["config"] if head else {})),
            "roofline": head["roofline"] if head else None, "decode": decode,
            "e2e": head.get("e2e") if head else None, "cpu_baseline": head.get("cpu_baseline") if head else None,
            "gpu_launches": head["gpu_launches"] if head else 0, "clocks": head["clocks"] if head else None,
        }
        line.update(extra)
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def gdn_tc_active(gdn, dev, w) -> bool:
    import torch
    major, _ = torch.cuda.get_device_capability()
    return major == 10 and w.dtype == "bf16" and w.d == 128 and w.chunk == 64 and tc_built(gdn)


def backward_tc_active(gdn, dev, w) -> bool:
    """The backward takes the tensor-core kernels (bf16, d = 128, sm_100)."""
    import torch
    major, _ = torch.cuda.get_device_capability()
    return major == 10 and w.dtype == "bf16" and w.d == 128 and w.hv % w.hk == 0


def tc_built(gdn) -> bool:
    src = open(os.path.join(ROOT, "linear_attention_sequence_sm_b200", "csrc", "gdn_chunk_tc.cu")).read()
    return "tcgen05.mma" in src


def useful_flops_per_vhead_token(group: int, d: int = 128, chunk: int = 64) -> int:
    """6 d^2 (inter-chunk) + 3 C d (triangular intra-chunk, counted at half)
    + 2 C d / G (the Gram shared by the G value heads of a q/k head)."""
    return 6 * d * d + 3 * chunk * d + 2 * chunk * d // group


FP32_LANES_PER_SM = 128


def backward_flops_per_vhead_token(d: int = 128, chunk: int = 64) -> int:
    """Useful flops of the tensor-core backward per (token, value head), every
    product counted once (not the two or three instructions its split
    operands take): the factors (K K^T, Q K^T, W, U~, P W: C x C x d each;
    (W diag(lambda))^T K: d x d x C), the two chains (S M', dS M'^T: d x d x d;
    U~^T diag(lambda) K, dO^T X: d x d x C), and the gradients (five
    C x d x d products, thirteen C x C x d, two C x C x C):
    36 C^2 d + 16 C d^2 + 4 d^3 + 4 C^3 per chunk."""
    C = chunk
    return (36 * C * C * d + 16 * C * d * d + 4 * d ** 3 + 4 * C ** 3) // C


def kda_flops_per_vhead_token(d: int = 128) -> int:
    """Kimi Delta Attention in token order: per state element a decay
    multiply, two dot-product FMAs (s'.k, s'.q) and the rank-1 write FMA."""
    return 7 * d * d


def prefill_bytes(w, kda: bool = False) -> int:
    """Mandatory HBM bytes of one prefill: q, k, v, o once, g and beta, the
    initial state (if any) and the final state (KDA: g per key channel)."""
    esz = 2 if w.dtype == "bf16" else 4
    t = w.total_tokens
    b = t * w.hk * w.d * esz * 2 + t * w.hv * w.d * esz * 2 + t * w.hv * (4 * w.d + 4 if kda else 8)
    b += w.num_seqs * w.hv * w.d * w.d * 4 * (2 if w.s0_std > 0 else 1)
    return b


def conv_bytes(w, width: int) -> int:
    """Algorithmic bytes of one --conv step: q, k and v read and written once
    in the storage dtype, the fp32 filters read, the fp32 conv states written."""
    es = 2 if w.dtype == "bf16" else 4
    ch = 2 * w.hk * w.d + w.hv * w.d
    return w.total_tokens * ch * es * 2 + ch * width * 4 + w.num_seqs * ch * (width - 1) * 4


def decode_bytes(dw, kda: bool = False, mtp: int = 0) -> int:
    """Bytes one decode step must move: the fp32 state read and written once,
    plus q, k, v, o (bf16) and g, beta (fp32; KDA: g per key channel).  With
    mtp = K draft tokens: the state read once and K snapshots written, and K
    tokens' inputs and outputs."""
    s = dw.num_seqs * dw.hv * dw.d * dw.d * 4
    gb = dw.hv * (4 * dw.d + 4) if kda else 2 * dw.hv * 4
    per_tok = dw.num_seqs * (2 * dw.hk * dw.d * 2 + 2 * dw.hv * dw.d * 2 + gb)
    if mtp > 0:
        return s * (1 + mtp) + per_tok * mtp
    return 2 * s + per_tok


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
