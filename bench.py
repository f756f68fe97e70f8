"""Benchmark of the DARKformer PRF attention forward pass on B200.

Default workload: the large-head causal forward, bf16, B=4 H=8 L=8192 d=256
r=256 m=512 with orthogonal features and anisotropic queries and keys (the
largest single-GPU configuration of the method's forward path; seeded
synthetic inputs), followed by the streaming decode step (B=64 H=8 d=64
m=256 after a 4096-token prefill), reported under the key "decode".

One JSON line on rank 0. `value` is whole-job forward tokens/s (B*H*L per
step, summed over ranks) with inputs resident in HBM and L2 flushed before
every timed step; `e2e` is the same metric through the C ABI with pinned host
buffers, host->device and device->host copies inside the timed region.
`--impl reference` times the fp64 CPU oracle on the host cores instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch
import torch.distributed as dist

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from random_feature_linear_b200 import synth  # noqa: E402

L2_FLUSH_BYTES = 512 << 20        # > 126 MB L2
L2_CLEAN_BYTES = 256 << 20
L2_NOTE = ("flushed before every timed step: 512 MiB written, then 256 MiB of other data read "
           "(no line of the step's data and no dirty line left in L2)")


class L2Flush:
    """Writes a buffer larger than L2, then reads a second one: the write evicts
    every line the timed call could reuse, the read leaves L2 holding clean
    lines, so that writing back the flush's own dirty lines is not charged to
    the next timed call."""

    def __init__(self, dev):
        self.w = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
        self.r = torch.zeros(L2_CLEAN_BYTES // 4, dtype=torch.int32, device=dev)

    def __call__(self):
        self.w.zero_()
        self.r.sum()


METRIC = "DARK attention fwd tokens/s (B\u00b7H\u00b7L/s) on 1 B200; % of BF16-tensor/HBM roofline"

# DRAM bytes (read + write) per forward call from one ncu capture per kernel
# of the call, summed over its launches: the large-head causal workload
# (B4 H8 L8192 d256 r256 m512; features_kernel 271.8 + 552.4 MB, values_kernel
# 744.6 + 117.9 MB). Reported only while the kernel sources hash to what was
# captured.
_NCU_TRAFFIC = {
    4: (("tc_wide.cu", "tc_common.cuh", "common.cuh", "internal.h", "tc_roles.cuh"),
        "6615388094732260", 271.751936e6 + 552.398080e6 + 744.621312e6 + 117.852160e6),
}


def captured_traffic(cfg: int):
    if cfg not in _NCU_TRAFFIC:
        return None
    sources, digest, nbytes = _NCU_TRAFFIC[cfg]
    h = hashlib.sha256()
    for f in sources:
        with open(os.path.join(ROOT, "random_feature_linear_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return nbytes if h.hexdigest()[:16] == digest else None


# Nominal exp2 rate of the special-function units: 16 per clock per SM x 148
# SMs x 1.965 GHz (an explanatory third bound next to tensor and HBM time).
MUFU_EX2_PER_S = 16 * 148 * 1.965e9


def max_over_ranks(value: float, device) -> float:
    """The largest of every rank's value (the job's time is its slowest rank's);
    the value itself on one rank or without a process group."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


E2E_NOTE = ("pinned host buffers, double-buffered over three streams (one stream when a "
            "step moves under 4 MiB): step i's host-to-device copies overlap step i-1's call "
            "and its device-to-host copies; every step copies all of its inputs in and its "
            "outputs out; time from the first copy in to the last copy out")
E2E_OVERLAP_MIN_BYTES = 4 << 20


def pipelined_e2e(host_in, dev_in_like, call, dev_out_like, host_out, steps: int, warmup: int,
                  dev) -> float:
    """Milliseconds per step of `steps` end-to-end steps through the public
    call: the inputs of step i (host_in(i), pinned) are copied in on one
    stream, `call(inputs, outputs)` runs on a second, the outputs are copied
    back into `host_out` (pinned) on a third, with two device buffer sets so
    that the copies of neighbouring steps overlap the call (PCIe carries both
    directions at once). Events order each buffer set's reuse. A step that
    moves less than E2E_OVERLAP_MIN_BYTES runs all three parts on one stream:
    there the cross-stream waits cost more than the overlap saves."""
    moved = sum(t.numel() * t.element_size() for t in list(dev_in_like) + list(dev_out_like))
    if moved < E2E_OVERLAP_MIN_BYTES:
        s_in = s_cmp = s_out = torch.cuda.Stream(device=dev)
    else:
        s_in, s_cmp, s_out = (torch.cuda.Stream(device=dev) for _ in range(3))
    ins = [[torch.empty_like(t) for t in dev_in_like] for _ in range(2)]
    outs = [[torch.empty_like(t) for t in dev_out_like] for _ in range(2)]
    ev_in, ev_cmp, ev_out = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))

    def step(i):
        k = i % 2
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_cmp[k])      # the call two steps back has read set k
            for d, h in zip(ins[k], host_in(i)):
                d.copy_(h, non_blocking=True)
            ev_in[k].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(ev_in[k])
            s_cmp.wait_event(ev_out[k])     # the copy out two steps back has read set k
            call(ins[k], outs[k])
            ev_cmp[k].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_cmp[k])
            for h, d in zip(host_out, outs[k]):
                h.copy_(d, non_blocking=True)
            ev_out[k].record(s_out)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(steps):
        step(i)
    e1.record(s_out)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def alg_flops(w: synth.Workload) -> float:
    """Algorithmic FLOPs of one forward pass: per head 2Ldm (query features) +
    2Ld(m+r) (key features and norms) + 2Lm(d+1) (state) + 2Lm(d+1) (output)."""
    per_head = (2 * w.L * w.d * w.m + 2 * w.L * w.d * (w.m + w.r) + 4 * w.L * w.m * (w.d + 1))
    return float(per_head * w.B * w.H)


def alg_bytes(w: synth.Workload) -> float:
    """Algorithmic HBM bytes: q, k, v read and out written once, plus the mask."""
    elt = 2 if w.dtype == "bf16" else 4
    return float(4 * w.B * w.H * w.L * w.d * elt + (w.B * w.L if w.lengths else 0))


def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], source="measured")
    return dict(hbm=6650.0, bf16=1590.0, source="fallback")


class ClockSampler:
    """Polls SM clock and clock-event (throttle) reasons through NVML every
    ~1 ms while the timed region runs (a background thread)."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, cuda_index: int):
        self.samples = []
        self.max_mhz = None
        self.stop = threading.Event()
        self.thread = None
        self.handle = None
        try:
            import pynvml
            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
            ids = [x for x in vis.split(",") if x.strip() != ""]
            idx = int(ids[cuda_index]) if ids and ids[cuda_index].strip().isdigit() else cuda_index
            self.nvml = pynvml
            self.handle = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.handle = None

    def _reasons(self) -> int:
        f = getattr(self.nvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(self.nvml, "nvmlDeviceGetCurrentClocksThrottleReasons")
        return int(f(self.handle))

    def _run(self):
        while not self.stop.is_set():
            try:
                mhz = self.nvml.nvmlDeviceGetClockInfo(self.handle, self.nvml.NVML_CLOCK_SM)
                self.samples.append((mhz, self._reasons()))
            except Exception:
                pass
            time.sleep(0.001)

    def __enter__(self):
        if self.handle is not None:
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=2)

    def summary(self) -> dict:
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"], "samples": 0}
        mhz = [m for m, _ in self.samples]
        bits = 0
        for _, r in self.samples:
            bits |= r
        reasons = sorted(name for bit, name in self.REASONS.items() if bits & bit)
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(self.samples)}


def oracle_sample(w: synth.Workload, inp: dict, max_seconds: float = 20.0, exact: bool = False):
    """Times the fp64 oracle on whole (batch, head) slices of the workload until
    about `max_seconds` of CPU work; returns (tokens/s, tokens, seconds, heads)."""
    from oracle import dark_oracle as O
    done_tokens, t_total, heads = 0, 0.0, 0
    for b in range(w.B):
        for h in range(w.H):
            sl = (slice(b, b + 1), slice(h, h + 1))
            geom = inp["geom"][h:h + 1] if inp["geom"].shape[0] > 1 else inp["geom"]
            mask = None if inp["mask"] is None else inp["mask"][b:b + 1]
            t0 = time.perf_counter()
            if exact:
                O.exact_attention(inp["q"][sl], inp["k"][sl], inp["v"][sl], geom,
                                  key_mask=mask, causal=w.causal)
            else:
                O.attention(inp["q"][sl], inp["k"][sl], inp["v"][sl], inp["omega"], geom,
                            key_mask=mask, causal=w.causal)
            t_total += time.perf_counter() - t0
            done_tokens += w.L
            heads += 1
            if t_total > max_seconds:
                return done_tokens / t_total, done_tokens, t_total, heads
    return done_tokens / t_total, done_tokens, t_total, heads


def host_cores() -> int:
    """Cores this process may run on (its CPU affinity set)."""
    return len(os.sched_getaffinity(0))


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


class oracle_threads:
    """Runs the oracle's numpy/BLAS work on every core of the affinity set, so
    that the reported core count is the thread count actually used."""

    def __enter__(self):
        self.n = host_cores()
        self.ctl = None
        try:
            from threadpoolctl import threadpool_limits
            self.ctl = threadpool_limits(limits=self.n)
        except Exception:
            self.ctl = None
        return self

    def __exit__(self, *exc):
        if self.ctl is not None:
            self.ctl.restore_original_limits()


def cpu_info(n: int) -> dict:
    return {"cores": n, "cpu_model": cpu_model()}


def count_launches(fn) -> tuple[int, list]:
    """Kernels of the native library launched by one call of fn (CUPTI via torch.profiler)."""
    from torch.profiler import ProfilerActivity, profile
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        fn()
        torch.cuda.synchronize()
    names = [e.name for e in prof.events() if e.device_type == torch.autograd.DeviceType.CUDA]
    ours = [n for n in names if "dark::" in n]
    return len(ours), sorted(set(ours))


def run_native(args, w: synth.Workload, rank: int, world: int, dev) -> dict | None:
    from random_feature_linear_b200 import dark as D
    inp = synth.make_inputs(w, salt=rank)
    dt = D.DARK_BF16 if w.dtype == "bf16" else D.DARK_F32
    tdt = D.torch_dtype(dt)
    omega = torch.from_numpy(inp["omega"]).to(dev)
    geom = torch.from_numpy(inp["geom"]).to(dev)
    proj, _wbuf = D.dark_make_projection(omega, geom, w.H, dt)
    q, k, v = (torch.from_numpy(inp[n]).to(dev).to(tdt) for n in ("q", "k", "v"))
    mask = None if inp["mask"] is None else torch.from_numpy(inp["mask"]).to(dev)
    out = torch.empty_like(q)
    flags = (D.DARK_CAUSAL if w.causal else 0) | (D.DARK_EXACT if args.exact else 0) | \
        (D.DARK_STABILISE if args.stabilise else 0)
    ws = D.alloc_workspace(proj, w.B, w.H, w.L, flags, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = None if args.ncu else L2Flush(dev)
    stream = torch.cuda.current_stream()

    def step():
        D.dark_attention_fwd(proj, q, k, v, out, w.B, w.H, w.L, key_mask=mask, flags=flags,
                             ws=ws, dev_status=status)

    if args.ncu:
        # capture mode for Nsight Compute: the forward calls only (ncu flushes
        # caches itself before every replayed kernel)
        for _ in range(args.warmup + args.steps):
            step()
        torch.cuda.synchronize()
        assert int(status.item()) == 0, D.dark_status_string(int(status.item()))
        return None
    for _ in range(args.warmup):
        flush()
        step()
    torch.cuda.synchronize()
    # The timed forward is one replay of a CUDA graph holding the API call's
    # launches, so host-side argument checks and descriptor encoding do not
    # leave the device idle between them (the e2e figure below keeps them).
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        step()
        side.synchronize()
        with torch.cuda.graph(graph, stream=side):
            step()
    stream.wait_stream(side)
    torch.cuda.synchronize()
    if args.no_profile:
        launches_per_step, kernel_names = 1, ["(not counted: --no-profile)"]
    else:
        launches_per_step, kernel_names = count_launches(step)

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        wall0 = time.perf_counter()
        for i in range(args.steps):
            flush()                       # L2 flush, outside the timed interval
            starts[i].record(stream)
            graph.replay()
            ends[i].record(stream)
        torch.cuda.synchronize()
        wall = time.perf_counter() - wall0
    if world > 1:
        dist.barrier()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    ms_per_step = max_over_ranks(sum(step_ms), dev) / args.steps
    assert int(status.item()) == 0, D.dark_status_string(int(status.item()))

    # end to end through the C ABI with pinned host buffers
    srcs = [q, k, v] + ([] if mask is None else [mask])
    host = [t.cpu().pin_memory() for t in srcs]
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()

    def e2e_call(ins, outs):
        D.dark_attention_fwd(proj, ins[0], ins[1], ins[2], outs[0], w.B, w.H, w.L,
                             key_mask=ins[3] if mask is not None else None, flags=flags,
                             ws=ws, dev_status=status)

    if world > 1:
        dist.barrier()
    e2e_ms = max_over_ranks(pipelined_e2e(lambda i: host, srcs, e2e_call, [out], [hout],
                                          args.steps, args.warmup, dev), dev)
    assert int(status.item()) == 0, D.dark_status_string(int(status.item()))
    h2d = sum(t.numel() * t.element_size() for t in host)
    d2h = hout.numel() * hout.element_size()

    if rank != 0:
        return None
    tokens = w.tokens * world
    peaks = load_peaks()
    t_kernel = ms_per_step / 1e3            # the whole forward call (its launches back to back)
    flops = alg_flops(w)
    nbytes = alg_bytes(w)
    t_tc = flops / (peaks["bf16"] * 1e12)
    t_hbm = nbytes / (peaks["hbm"] * 1e9)
    if args.exact:
        flops = exact_flops(w)
        achieved = flops / t_kernel / 1e12
        if w.dtype == "bf16" and w.d == 64 and w.r % 16 == 0 and w.r <= 64:
            roof = dict(bound="tensor", achieved=achieved, peak=peaks["bf16"], unit="TFLOP/s",
                        frac=achieved / peaks["bf16"], traffic=None,
                        peak_source=peaks["source"] + " (burst)",
                        kernel="exact-mode call (exact_tc_kernel, tcgen05)")
        else:
            roof = dict(bound="alu", achieved=achieved, peak=FFMA_TFLOPS, unit="TFLOP/s",
                        frac=achieved / FFMA_TFLOPS, traffic=None,
                        peak_source="derived: 148 SMs x 128 FP32 lanes x 2 x 1.965 GHz",
                        kernel="exact-mode call (SIMT fp32)")
    else:
        bound = "tensor" if t_tc >= t_hbm else "hbm"
        if bound == "tensor":
            achieved = flops / t_kernel / 1e12
            roof = dict(bound="tensor", achieved=achieved, peak=peaks["bf16"], unit="TFLOP/s",
                        frac=achieved / peaks["bf16"], traffic=None)
        else:
            achieved = nbytes / t_kernel / 1e9
            roof = dict(bound="hbm", achieved=achieved, peak=peaks["hbm"], unit="GB/s",
                        frac=achieved / peaks["hbm"], traffic=None)
        roof["peak_source"] = peaks["source"] + " (burst)"
        short = sorted({k.replace("(anonymous namespace)::", "").split("(")[0].split("<")[0].split("::")[-1]
                        for k in kernel_names if "dark::" in k})
        roof["kernel"] = "forward call" + (" (" + ", ".join(short) + ")" if short else "")
        # the capture is of the plain call's kernels (not the stabilised one)
        roof["traffic"] = None if args.stabilise else captured_traffic(args.workload)
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        with oracle_threads() as ot:
            tps, ntok, secs, heads = oracle_sample(w, inp, exact=args.exact)
        cpu = dict(value=tps, unit="tokens/s", kind="oracle", **cpu_info(ot.n),
                   sample=f"{heads} of {w.B * w.H} (batch, head) slices, {ntok} tokens, {secs:.1f} s")
    clocks = clk.summary()
    return {
        "metric": EXACT_METRIC if args.exact else METRIC,
        "value": tokens / (ms_per_step / 1e3),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic (seeded numpy, orthogonal Gaussian features)",
        "config": {"workload": ("exact mode: " if args.exact else "") +
                               ("stabilised: " if args.stabilise else "") + w.name,
                   "B": w.B, "H": w.H,
                   "L": w.L, "d": w.d, "r": w.r, "m": w.m,
                   "causal": w.causal, "lengths": list(w.lengths) if w.lengths else None,
                   "l2": L2_NOTE,
                   "timing": "CUDA events around one CUDA-graph replay of the forward call per step",
                   "parallelism": f"replicas x{world} (independent batches, no collective)"},
        "e2e": {"value": tokens / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "how": E2E_NOTE},
        "roofline": roof,
        "roofline_other": {"t_tensor_us": t_tc * 1e6, "t_hbm_us": t_hbm * 1e6,
                           "t_mufu_us_nominal": 2.0 * w.tokens * w.m / MUFU_EX2_PER_S * 1e6,
                           "alg_flops": flops, "alg_bytes": nbytes},
        "cpu_baseline": cpu,
        "gpu_launches": launches_per_step * args.steps,
        "kernels": kernel_names,
        "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"],
                   "reasons": clocks["reasons"], "samples": clocks["samples"]},
        "wall_s": wall,
        "step_ms_min": min(step_ms),
    }


DECODE_METRIC = "DARK decode step tokens/s (B\u00b7H rows per step) on 1 B200; % of HBM roofline"


def decode_bytes(w: synth.Workload) -> float:
    """Algorithmic HBM bytes of one decode step: the fp32 (KV, z) state read and
    written once, plus q, k, v in and out."""
    state = w.B * w.H * w.m * (w.d + 1) * 4
    io = 4 * w.B * w.H * w.d * (2 if w.dtype == "bf16" else 4)
    return 2 * state + io


def oracle_decode_sample(w: synth.Workload, kv, z, stream, omega, geom, max_seconds: float = 10.0):
    """Times fp64 oracle decode steps over all (batch, head) slices; returns
    (rows/s, steps done, seconds)."""
    from oracle import dark_oracle as O
    done, t_total = 0, 0.0
    while t_total < max_seconds and done < stream["q"].shape[0]:
        t0 = time.perf_counter()
        _, kv, z = O.decode_step(kv, z, stream["q"][done], stream["k"][done], stream["v"][done],
                                 omega, geom)
        t_total += time.perf_counter() - t0
        done += 1
    return done * w.B * w.H / t_total, done, t_total


def run_decode(args, rank: int, world: int, dev) -> dict | None:
    """Streaming decode (workload 5): a causal prefill fills the (KV, z) state
    outside the timed region; each timed iteration is one decode step replayed
    from a CUDA graph, with the L2 flushed before it (the state then comes from
    HBM). A 1024-step graph, state L2-warm, is reported beside it."""
    from random_feature_linear_b200 import dark as D
    w = synth.WORKLOADS[5]
    inp = synth.make_inputs(w, salt=rank)
    dt = D.DARK_BF16
    omega = torch.from_numpy(inp["omega"]).to(dev)
    geom = torch.from_numpy(inp["geom"]).to(dev)
    proj, _wbuf = D.dark_make_projection(omega, geom, w.H, dt)
    q, k, v = (torch.from_numpy(inp[n]).to(dev).to(torch.bfloat16) for n in ("q", "k", "v"))
    out = torch.empty_like(q)
    st, st_t = D.make_state(proj, w.B, w.H, dev)
    ws = D.alloc_workspace(proj, w.B, w.H, w.L, D.DARK_CAUSAL, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    D.dark_attention_fwd(proj, q, k, v, out, w.B, w.H, w.L, flags=D.DARK_CAUSAL, state_out=st,
                         ws=ws, dev_status=status)
    n_graph = 1024
    stream_np = synth.decode_stream(w, n_graph, salt=rank)
    sq, sk, sv = (torch.from_numpy(stream_np[n]).to(dev).to(torch.bfloat16) for n in ("q", "k", "v"))
    so = torch.empty_like(sq)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream()

    def one(i):
        D.dark_decode_step(proj, st, sq[i], sk[i], sv[i], so[i], dev_status=status)

    if args.ncu:
        # capture mode for Nsight Compute: warmup + steps decode calls only
        for i in range(args.warmup + args.steps):
            one(i % n_graph)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, D.dark_status_string(int(status.item()))
        return None
    for i in range(args.warmup):
        one(i)
    torch.cuda.synchronize()
    launches, kernel_names = (1, ["(not counted: --no-profile)"]) if args.no_profile else \
        count_launches(lambda: one(0))
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    g1, gall = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(g1, stream=side):
            one(0)
        with torch.cuda.graph(gall, stream=side):
            for i in range(n_graph):
                one(i)
    stream.wait_stream(side)
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        for i in range(args.steps):
            flush()
            starts[i].record(stream)
            g1.replay()
            ends[i].record(stream)
        torch.cuda.synchronize()
    step_ms = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    ms = statistics.median(step_ms)
    # 1024 consecutive steps in one graph (state stays in L2 between steps)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    gall.replay()
    torch.cuda.synchronize()
    e0.record(stream)
    gall.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    warm_ms = e0.elapsed_time(e1) / n_graph
    if int(status.item()) != 0:
        raise RuntimeError(D.dark_status_string(int(status.item())))
    # end to end: pinned host q, k, v in, the call, out back to the host, per step
    hq, hk, hv = (t[:args.steps].cpu().pin_memory() for t in (sq, sk, sv))
    ho = torch.empty_like(hq[0]).pin_memory()
    dq, do = sq[0], sq[0]

    def e2e_call(ins, outs):
        D.dark_decode_step(proj, st, ins[0], ins[1], ins[2], outs[0], dev_status=status)

    n_e2e = hq.shape[0]
    e2e_ms = max_over_ranks(pipelined_e2e(
        lambda i: [hq[i % n_e2e], hk[i % n_e2e], hv[i % n_e2e]], [sq[0], sk[0], sv[0]], e2e_call,
        [sq[0]], [ho], args.steps, 0, dev), dev)
    ms = max_over_ranks(ms, dev)
    if rank != 0:
        return None
    rows = w.B * w.H * world
    t = ms / 1e3
    peaks = load_peaks()
    nbytes = decode_bytes(w)
    achieved = nbytes / t / 1e9
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        kv0 = st_t[0][:1].double().cpu().numpy()
        z0 = st_t[1][:1].double().cpu().numpy()
        sub = {n: stream_np[n][:, :1] for n in ("q", "k", "v")}
        with oracle_threads() as ot:
            rps, nsteps, secs = oracle_decode_sample(w.with_sizes(B=1), kv0, z0, sub,
                                                     inp["omega"], inp["geom"])
        cpu = dict(value=rps, unit="tokens/s", kind="oracle", **cpu_info(ot.n),
                   sample=f"batch row 0 ({w.H} heads), {nsteps} decode steps, {secs:.1f} s")
    clocks = clk.summary()
    return {
        "metric": DECODE_METRIC, "value": rows / t, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded numpy, orthogonal Gaussian features)",
        "config": {"workload": "decode after a 4096-token causal prefill (B64 H8 d64 r64 m256, "
                               "fp32 state)", "B": w.B, "H": w.H, "d": w.d, "r": w.r, "m": w.m,
                   "l2": L2_NOTE,
                   "timing": "CUDA events around a one-step CUDA-graph replay",
                   "parallelism": f"replicas x{world} (independent batches, no collective)"},
        "e2e": {"value": rows / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": 3 * dq.numel() * dq.element_size(),
                "d2h_bytes_per_step": do.numel() * do.element_size(), "how": E2E_NOTE},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm"], "traffic": None,
                     "peak_source": peaks["source"], "kernel": "decode step (decode_pair_kernel for this workload)"},
        "warm_graph_1024": {"ms_per_step": warm_ms, "value": rows / (warm_ms / 1e3),
                            "GBps_algorithmic": nbytes / (warm_ms / 1e3) / 1e9,
                            "note": "state L2-resident between steps"},
        "cpu_baseline": cpu,
        "gpu_launches": launches * args.steps,
        "kernels": kernel_names,
        "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"],
                   "reasons": clocks["reasons"], "samples": clocks["samples"]},
    }


CROSS_METRIC = ("DARK cross-attention fwd tokens/s (B·H·(Lq+Lk)/s) on 1 B200; "
                "% of BF16-tensor/HBM roofline")
CROSS_LQ, CROSS_LK = 256, 1024


def cross_workload() -> synth.Workload:
    """The README's cross-attention example (8 heads of 64, 256 features, 256
    queries over 1024 context tokens, batch 2) with the causal recipe's draws."""
    return synth.WORKLOADS[2].with_sizes(B=2, H=8, L=CROSS_LQ, causal=False, lengths=None)


def cross_flops_bytes(w: synth.Workload, lq: int, lk: int) -> tuple[float, float]:
    """Per head 2 Lq d m (query features) + 2 Lk d (m+r) (context features and
    norms) + 2 Lk m (d+1) (summary) + 2 Lq m (d+1) (output); bytes: q and out
    over Lq tokens, k and v over Lk tokens, once each, plus both masks."""
    per_head = 2 * lq * w.d * w.m + 2 * lk * w.d * (w.m + w.r) + 2 * (lq + lk) * w.m * (w.d + 1)
    elt = 2 if w.dtype == "bf16" else 4
    nbytes = 2 * w.B * w.H * (lq + lk) * w.d * elt + w.B * (lq + lk)
    return float(per_head * w.B * w.H), float(nbytes)


def run_cross(args, rank: int, world: int, dev) -> dict | None:
    """Cross-attention forward of queries over a separate context (both masks
    given, all valid as in the README example); timed like the self-attention
    forward: one CUDA-graph replay per step, L2 flushed before each."""
    from random_feature_linear_b200 import dark as D
    w, lq, lk = cross_workload(), CROSS_LQ, CROSS_LK
    iq = synth.make_inputs(w, salt=rank)
    ik = synth.make_inputs(w.with_sizes(L=lk), salt=rank + 1000)
    tdt = D.torch_dtype(D.DARK_BF16)
    proj, _wbuf = D.dark_make_projection(torch.from_numpy(iq["omega"]).to(dev),
                                         torch.from_numpy(iq["geom"]).to(dev), w.H, D.DARK_BF16)
    q = torch.from_numpy(iq["q"]).to(dev).to(tdt)
    k, v = (torch.from_numpy(ik[n]).to(dev).to(tdt) for n in ("k", "v"))
    qm = torch.ones(w.B, lq, dtype=torch.uint8, device=dev)
    cm = torch.ones(w.B, lk, dtype=torch.uint8, device=dev)
    out = torch.empty_like(q)
    ws = D.alloc_cross_workspace(proj, w.B, w.H, lq, lk, 0, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream()

    def call(q_, k_, v_, qm_, cm_, out_=None):
        D.dark_cross_attention_fwd(proj, q_, k_, v_, out if out_ is None else out_, w.B, w.H, lq,
                                   lk, query_mask=qm_, context_mask=cm_, ws=ws, dev_status=status)

    for _ in range(args.warmup):
        flush()
        call(q, k, v, qm, cm)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        call(q, k, v, qm, cm)
        side.synchronize()
        with torch.cuda.graph(graph, stream=side):
            call(q, k, v, qm, cm)
    stream.wait_stream(side)
    torch.cuda.synchronize()
    launches_per_step, kernel_names = (1, ["(not counted: --no-profile)"]) if args.no_profile \
        else count_launches(lambda: call(q, k, v, qm, cm))
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        for i in range(args.steps):
            flush()
            starts[i].record(stream)
            graph.replay()
            ends[i].record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms_per_step = max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(starts, ends)), dev) \
        / args.steps
    assert int(status.item()) == 0, D.dark_status_string(int(status.item()))

    srcs = [q, k, v, qm, cm]
    host = [t.cpu().pin_memory() for t in srcs]
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    if world > 1:
        dist.barrier()
    e2e_ms = max_over_ranks(pipelined_e2e(lambda i: host, srcs, lambda ins, outs: call(*ins, out_=outs[0]),
                                          [out], [hout], args.steps, args.warmup, dev), dev)
    if rank != 0:
        return None
    tokens = w.B * w.H * (lq + lk) * world
    peaks = load_peaks()
    flops, nbytes = cross_flops_bytes(w, lq, lk)
    t = ms_per_step / 1e3
    t_tc, t_hbm = flops / (peaks["bf16"] * 1e12), nbytes / (peaks["hbm"] * 1e9)
    if t_tc >= t_hbm:
        roof = dict(bound="tensor", achieved=flops / t / 1e12, peak=peaks["bf16"], unit="TFLOP/s")
    else:
        roof = dict(bound="hbm", achieved=nbytes / t / 1e9, peak=peaks["hbm"], unit="GB/s")
    roof.update(frac=roof["achieved"] / roof["peak"], traffic=None,
                peak_source=peaks["source"] + " (burst)", kernel="cross-attention forward call")
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        from oracle import dark_oracle as O
        qn, kn, vn = iq["q"], ik["k"], ik["v"]
        with oracle_threads() as ot:
            t0, heads = time.perf_counter(), 0
            for b in range(w.B):
                for h in range(w.H):
                    sl = (slice(b, b + 1), slice(h, h + 1))
                    O.cross_attention(qn[sl], kn[sl], vn[sl], iq["omega"], iq["geom"][h:h + 1])
                    heads += 1
                    if time.perf_counter() - t0 > 10.0:
                        break
                else:
                    continue
                break
            secs = time.perf_counter() - t0
        cpu = dict(value=heads * (lq + lk) / secs, unit="tokens/s", **cpu_info(ot.n),
                   kind="oracle", sample=f"{heads} of {w.B * w.H} (batch, head) slices, {secs:.1f} s")
    clocks = clk.summary()
    return {
        "metric": CROSS_METRIC, "value": tokens / t, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded numpy, orthogonal Gaussian features)",
        "config": {"workload": f"cross-attention bf16 (B{w.B} H{w.H} Lq{lq} Lk{lk} d{w.d} r{w.r} "
                               f"m{w.m}, all-valid query and context masks)",
                   "l2": L2_NOTE,
                   "timing": "CUDA events around one CUDA-graph replay of the forward call per step",
                   "parallelism": f"replicas x{world} (independent batches, no collective)"},
        "e2e": {"value": tokens / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": sum(x.numel() * x.element_size() for x in host),
                "d2h_bytes_per_step": hout.numel() * hout.element_size(), "how": E2E_NOTE},
        "roofline": roof,
        "roofline_other": {"t_tensor_us": t_tc * 1e6, "t_hbm_us": t_hbm * 1e6,
                           "alg_flops": flops, "alg_bytes": nbytes},
        "cpu_baseline": cpu,
        "gpu_launches": launches_per_step * args.steps,
        "kernels": kernel_names,
        "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"],
                   "reasons": clocks["reasons"], "samples": clocks["samples"]},
    }


EXACT_METRIC = ("DARK exact learned-kernel attention fwd tokens/s (B·H·L/s) on 1 B200; "
                "% of BF16-tensor roofline (tcgen05 path) or FP32-FFMA (SIMT path)")


def exact_flops(w: synth.Workload) -> float:
    """Exact mode per head: projections 2·2Ldr, then per visible (query, key) pair
    2r (score) + 2d (P V); L^2/2 pairs when causal."""
    pairs = w.L * (w.L + 1) / 2 if w.causal else w.L * w.L
    return float((4 * w.L * w.d * w.r + pairs * 2 * (w.r + w.d)) * w.B * w.H)


BWD_METRIC = ("DARK attention bwd tokens/s (B·H·L/s, dq dk dv dM) on 1 B200; "
              "% of TF32-tensor roofline (bf16 I/O) or FP32-FFMA (fp32 I/O)")
# fp32 FFMA peak: 148 SMs x 128 lanes x 2 FLOP x 1.965 GHz (the fp32-I/O backward
# kernels are SIMT fp32 throughout)
FFMA_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12
# dense tf32 / bf16 tensor throughput, nominal (1.1 and 2.25 PFLOP/s): the tf32
# peak is the measured bf16 peak times this ratio
TF32_OVER_BF16 = 1.1 / 2.25


def bwd_flops(w: synth.Workload) -> float:
    """Algorithmic FLOPs of one backward pass, per head: features 2Ldm (queries)
    + 2Ld(m+r) (keys); five m x (d+1) contractions over L (forward statistics,
    [num | den], dphi(q), gradient statistics, dv with dphi(k)); dx 2Ldm +
    2Ld(m+r) + 2Ldr (key norms); dW' 4L(m+r)d. Causal diagonal tiles excluded."""
    L, d, m, r = w.L, w.d, w.m, w.r
    per_head = (2 * L * d * m + 2 * L * d * (m + r) + 5 * 2 * L * m * (d + 1)
                + 2 * L * d * m + 2 * L * d * (m + r) + 2 * L * d * r + 4 * L * (m + r) * d)
    return float(per_head * w.B * w.H)


def run_backward(args, w: synth.Workload, rank: int, world: int, dev) -> dict | None:
    """Backward pass of the workload's attention (gradients of q, k, v and M for
    a seeded upstream gradient); timed like the forward."""
    from random_feature_linear_b200 import dark as D
    inp = synth.make_inputs(w, salt=rank)
    dout_np = synth.make_cotangent(w, salt=rank)
    dt = D.DARK_BF16 if w.dtype == "bf16" else D.DARK_F32
    tdt = D.torch_dtype(dt)
    omega = torch.from_numpy(inp["omega"]).to(dev)
    geom = torch.from_numpy(inp["geom"]).to(dev)
    q, k, v = (torch.from_numpy(inp[n]).to(dev).to(tdt) for n in ("q", "k", "v"))
    g = torch.from_numpy(dout_np).to(dev).to(tdt)
    mask = None if inp["mask"] is None else torch.from_numpy(inp["mask"]).to(dev)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    dgeom = torch.empty_like(geom)
    flags = D.DARK_CAUSAL if w.causal else 0
    ws = D.alloc_bwd_workspace(omega, geom, w.B, w.H, w.L, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream()

    def call(q_, k_, v_, g_, m_, outs_=None):
        o = (dq, dk, dv, dgeom) if outs_ is None else outs_
        D.dark_attention_bwd(omega, geom, q_, k_, v_, g_, o[0], o[1], o[2], w.B, w.H, w.L, dt,
                             key_mask=m_, flags=flags, dgeom=o[3], ws=ws, dev_status=status)

    if args.ncu:
        # capture mode for Nsight Compute: warmup + steps backward calls only
        for _ in range(args.warmup + args.steps):
            call(q, k, v, g, mask)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, D.dark_status_string(int(status.item()))
        return None
    for _ in range(args.warmup):
        flush()
        call(q, k, v, g, mask)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, D.dark_status_string(int(status.item()))
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        call(q, k, v, g, mask)
        side.synchronize()
        with torch.cuda.graph(graph, stream=side):
            call(q, k, v, g, mask)
    stream.wait_stream(side)
    torch.cuda.synchronize()
    launches_per_step, kernel_names = (1, ["(not counted: --no-profile)"]) if args.no_profile \
        else count_launches(lambda: call(q, k, v, g, mask))
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        for i in range(args.steps):
            flush()
            starts[i].record(stream)
            graph.replay()
            ends[i].record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms_per_step = max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(starts, ends)), dev) \
        / args.steps

    srcs = [q, k, v, g] + ([] if mask is None else [mask])
    host = [t.cpu().pin_memory() for t in srcs]
    outs = [dq, dk, dv, dgeom]
    houts = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs]
    if world > 1:
        dist.barrier()
    e2e_ms = max_over_ranks(pipelined_e2e(
        lambda i: host, srcs,
        lambda ins, o: call(ins[0], ins[1], ins[2], ins[3], ins[4] if mask is not None else None,
                            outs_=o),
        outs, houts, args.steps, args.warmup, dev), dev)
    assert int(status.item()) == 0, D.dark_status_string(int(status.item()))
    if rank != 0:
        return None
    tokens = w.tokens * world
    t = ms_per_step / 1e3
    flops = bwd_flops(w)
    peaks = load_peaks()
    if any("tbf_" in n for n in kernel_names):
        tf32 = peaks["bf16"] * TF32_OVER_BF16
        roof = dict(bound="tensor", achieved=flops / t / 1e12, peak=tf32, unit="TFLOP/s",
                    frac=flops / t / 1e12 / tf32, traffic=None,
                    peak_source=f"{peaks['source']} bf16 x {TF32_OVER_BF16:.3f} "
                                "(nominal dense tf32 / bf16)",
                    kernel="backward call (tcgen05 kind::tf32)")
    else:
        roof = dict(bound="alu", achieved=flops / t / 1e12, peak=FFMA_TFLOPS, unit="TFLOP/s",
                    frac=flops / t / 1e12 / FFMA_TFLOPS, traffic=None,
                    peak_source="derived: 148 SMs x 128 FP32 lanes x 2 x 1.965 GHz",
                    kernel="backward call (SIMT fp32)")
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        from oracle import dark_oracle as O
        with oracle_threads() as ot:
            t0, heads = time.perf_counter(), 0
            for h in range(w.H):
                sl = (slice(0, 1), slice(h, h + 1))
                gm = inp["geom"][h:h + 1] if inp["geom"].shape[0] > 1 else inp["geom"]
                O.attention_backward(inp["q"][sl], inp["k"][sl], inp["v"][sl], inp["omega"], gm,
                                     dout_np[sl], key_mask=None if inp["mask"] is None
                                     else inp["mask"][:1], causal=w.causal)
                heads += 1
                if time.perf_counter() - t0 > 10.0:
                    break
            secs = time.perf_counter() - t0
        cpu = dict(value=heads * w.L / secs, unit="tokens/s", **cpu_info(ot.n), kind="oracle",
                   sample=f"{heads} of {w.B * w.H} (batch, head) slices, {secs:.1f} s")
    clocks = clk.summary()
    return {
        "metric": BWD_METRIC, "value": tokens / t, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic (seeded numpy, orthogonal Gaussian features; dout ~ N(0,1))",
        "config": {"workload": "backward of " + w.name, "B": w.B, "H": w.H, "L": w.L, "d": w.d,
                   "r": w.r, "m": w.m, "causal": w.causal,
                   "l2": L2_NOTE,
                   "timing": "CUDA events around one CUDA-graph replay of the backward call per step",
                   "parallelism": f"replicas x{world} (independent batches, no collective)"},
        "e2e": {"value": tokens / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": sum(x.numel() * x.element_size() for x in host),
                "d2h_bytes_per_step": sum(x.numel() * x.element_size() for x in houts),
                "how": E2E_NOTE},
        "roofline": roof,
        "roofline_other": {"alg_flops": flops,
                           "frac_of_bf16_tensor_peak": flops / t / 1e12 / peaks["bf16"],
                           "t_ffma_us": flops / (FFMA_TFLOPS * 1e12) * 1e6},
        "cpu_baseline": cpu,
        "gpu_launches": launches_per_step * args.steps,
        "kernels": kernel_names,
        "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"],
                   "reasons": clocks["reasons"], "samples": clocks["samples"]},
    }


SAMPLE_METRIC = "DARK projection draw (orthogonal Omega, Philox4x64-10) draws/s on 1 B200"


def run_sample(args, rank: int, world: int, dev) -> dict | None:
    """Device draws of an orthogonal Omega for the causal workload's shape (m 256,
    r 64) and the large-head workload's (m 512, r 256): CUDA events around each
    draw (Gaussians, fp64 Gram-Schmidt per block, scaled rows)."""
    from random_feature_linear_b200 import dark as D
    res = {}
    launches = 0
    for name, m, r in (("m256 r64", 256, 64), ("m512 r256", 512, 256)):
        om = torch.empty(1, m, r, dtype=torch.float32, device=dev)
        ws = torch.empty(max(D.dark_sample_omega_workspace_bytes(1, m, r, True), 256),
                         dtype=torch.uint8, device=dev)
        for i in range(args.warmup):
            D.dark_sample_omega(1, i, om, ws=ws)
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        for i, (a, b) in enumerate(ev):
            a.record()
            D.dark_sample_omega(1, 1000 + i, om, ws=ws)
            b.record()
        torch.cuda.synchronize()
        ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev) / args.steps, dev)
        res[name] = ms
        launches += 3 * args.steps
    if rank != 0:
        return None
    main = res["m256 r64"]
    return {
        "metric": SAMPLE_METRIC, "value": world / (main / 1e3), "unit": "draws/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": main,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (counter-based generator)",
        "config": {"workload": "orthogonal Omega draw, m 256 r 64 (one head); also m 512 r 256",
                   "ms_per_draw": res,
                   "timing": "CUDA events around each draw; one draw per step"},
        "roofline": None,
        "gpu_launches": launches,
    }


def run_reference(args, w: synth.Workload) -> dict:
    inp = synth.make_inputs(w)
    with oracle_threads() as ot:
        for _ in range(args.warmup):
            oracle_sample(w, inp, max_seconds=1.0)
        vals, details = [], None
        for _ in range(args.steps):
            tps, ntok, secs, heads = oracle_sample(w, inp, max_seconds=args.ref_seconds)
            vals.append(tps)
            details = (ntok, secs, heads)
    value = statistics.median(vals)
    sample = f"{details[2]} of {w.B * w.H} (batch, head) slices per step, {details[0]} tokens"
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": value, "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": w.tokens / value * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded numpy, orthogonal Gaussian features)",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "L": w.L, "d": w.d, "r": w.r,
                   "m": w.m, "causal": w.causal},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "kind": "oracle",
                         "sample": sample, **cpu_info(ot.n)},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def decode_in_child(args) -> dict:
    """The decode line attached to a one-GPU forward run, measured by a fresh
    process (`bench.py --decode`): the CUDA profiler that counts launches
    records kernels in the first session of a process only."""
    import subprocess
    cmd = [sys.executable, os.path.abspath(__file__), "--decode", "--steps", str(args.steps),
           "--warmup", str(args.warmup)]
    cmd += ["--no-cpu-baseline"] if args.no_cpu_baseline else []
    cmd += ["--no-profile"] if args.no_profile else []
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    p = subprocess.run(cmd, capture_output=True, text=True, timeout=900, env=env)
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    if p.returncode != 0 or not lines:
        raise RuntimeError(f"decode run failed (rc {p.returncode}): {p.stderr[-2000:]}")
    return json.loads(lines[-1])


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", type=int, default=None,
                    help="synthetic workload recipe (1-5); default 4 for the forward, 2 for "
                         "--backward and --exact")
    ap.add_argument("--ref-seconds", type=float, default=None,
                    help="CPU seconds per reference step (default: about 120 s over all steps)")
    ap.add_argument("--no-decode", action="store_true",
                    help="leave the decode step out of the forward run's JSON line (it is "
                         "attached to one-GPU runs only)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-profile", action="store_true",
                    help="do not count launches with the CUDA profiler (for runs under ncu)")
    ap.add_argument("--decode", action="store_true",
                    help="time the streaming decode step (workload 5) instead of the forward")
    ap.add_argument("--stabilise", action="store_true",
                    help="forward with the overflow stabiliser (DARK_STABILISE)")
    ap.add_argument("--exact", action="store_true",
                    help="time the exact learned-kernel mode of --workload instead")
    ap.add_argument("--sample", action="store_true",
                    help="time device draws of an orthogonal projection instead")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward pass of --workload instead of the forward")
    ap.add_argument("--cross", action="store_true",
                    help="time cross-attention (256 queries over 1024 context tokens) instead")
    ap.add_argument("--ncu", action="store_true",
                    help="capture mode: only warmup + steps forward calls, no timing or output")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.ref_seconds is None:
        args.ref_seconds = max(1.0, min(10.0, 120.0 / max(args.steps + args.warmup, 1)))
    if args.workload is None:
        args.workload = 2 if (args.backward or args.exact) else 4
    w = synth.WORKLOADS[args.workload]

    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        # one process per GPU: relaunch this command under torchrun
        cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
               f"--nproc-per-node={args.gpus}", "--master-addr", "127.0.0.1",
               "--master-port", os.environ.get("MASTER_PORT", "29511"),
               os.path.abspath(__file__), *sys.argv[1:]]
        os.execv(sys.executable, cmd)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"bench.py: --gpus {args.gpus} but WORLD_SIZE is {world}; "
                         "launch one process per GPU (torchrun --nproc-per-node N)")
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, w)), flush=True)
        return
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    try:
        if args.decode:
            res = run_decode(args, rank, world, dev)
        elif args.cross:
            res = run_cross(args, rank, world, dev)
        elif args.backward:
            res = run_backward(args, w, rank, world, dev)
        elif args.sample:
            res = run_sample(args, rank, world, dev)
        else:
            res = run_native(args, w, rank, world, dev)
            if not (args.no_decode or args.ncu or args.exact) and world == 1:
                res["decode"] = decode_in_child(args)
        if res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
