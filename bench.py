"""Benchmark: exact attention forward + backward on one B200 per process.

A step is one pass of the whole hot path -- forward (fa_fwd_ws: V pass, persistent
kernel) then backward (fa_bwd_ws: preprocess reusing the forward's fp16 V, dK/dV kernel,
dQ kernel) -- over the causal workload
B=2, H=32, N=8192, d=128 (bf16 inputs, 1% of the keys of every head scaled by 8).
The metric is TFLOPS with 4*B*H*N^2*d forward flops (halved under the causal
mask) and 2.5x that for the backward.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (launched by torch.distributed.run) every rank runs an independent
replica of the workload on its own GPU (the method has no exchange step between
GPUs); the value is the total work of all ranks over the slowest rank's time.
``--impl reference`` times the fp64 CPU oracle on the host cores instead.
"""

from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from exact_io_aware_91_b200 import inputs  # noqa: E402

METRIC = "attention fwd/bwd TFLOPS (BF16, causal, N=8k, d=128) & % of B200 tensor peak"
WORKLOAD = 3  # the metric's workload; --workload picks another one for profiling only


KERNEL_OF = {"fwd": "fa_fwd_persist_sm100_kernel", "fwd_fp8": "fa_fwd_persist_sm100_kernel",
             "fwd_d256": "fa_fwd_d256_sm100_kernel", "bwd_dkdv": "fa_bwd_dkdv_sm100_kernel",
             "bwd_dq": "fa_bwd_dq_sm100_kernel"}
SHARED_HEADERS = ("sm100.cuh", "fa_internal.h")


def _strip_comments(text: str) -> str:
    """C++ source without its comments and blank lines (the kernel sources hold no comment
    markers inside string literals)."""
    import re

    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def kernel_source_digest(source: str, kernel_fn: str, text: str | None = None) -> str:
    """sha256 of the code a kernel can depend on: its source file with the bodies of the
    file's OTHER __global__ kernels removed, followed by the shared headers, all without
    comments.  A recorded ncu figure stays valid exactly while this digest is unchanged."""
    import hashlib
    import re

    csrc = os.path.join(ROOT, "exact_io_aware_91_b200", "csrc")
    if text is None:
        with open(os.path.join(csrc, source)) as f:
            text = f.read()
    text = _strip_comments(text)
    spans = []
    for mt in re.finditer(r"__global__\s+void\s+(?:__launch_bounds__\([^)]*\)\s*)?(\w+)\s*\(", text):
        if mt.group(1) == kernel_fn:
            continue
        i = text.index("{", mt.end())
        depth = 0
        for j in range(i, len(text)):
            depth += {"{": 1, "}": -1}.get(text[j], 0)
            if depth == 0:
                spans.append((i, j + 1))
                break
    kept, pos = [], 0
    for i, j in spans:
        kept.append(text[pos:i])
        pos = j
    kept.append(text[pos:])
    h = hashlib.sha256("".join(kept).encode())
    for name in SHARED_HEADERS:
        with open(os.path.join(csrc, name)) as f:
            h.update(_strip_comments(f.read()).encode())
    return h.hexdigest()


def recorded_traffic(kernel: str, workload_name: str):
    """DRAM bytes per launch from the committed ncu summary, if the kernel's code is unchanged."""
    short = {"causal_b2_h32_n8192_d128_spiky": "causal_b2_h32_n8192_d128",
             "causal_b2_h32_n8192_d128_spiky_fp8": "causal_b2_h32_n8192_d128_fp8",
             "causal_b2_h16_n8192_d256_spiky": "causal_b2_h16_n8192_d256",
             "causal_b4_h16_n2048_d128": "causal_b4_h16_n2048_d128",
             "noncausal_b64_h16_n512_d64": "noncausal_b64_h16_n512_d64"}.get(workload_name)
    if short is None:
        return None
    path = os.path.join(ROOT, "profiles", f"traffic_{short}.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(kernel)
    if not rec or "kernel_sha256" not in rec:
        return None
    if kernel_source_digest(rec["source"], rec.get("kernel_fn", KERNEL_OF[kernel])) != rec["kernel_sha256"]:
        return None  # the kernel (or code it depends on) changed since the counters were taken
    return rec["bytes"]


def load_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"bf16_tflops": d["bf16_tflops"], "bf16_tflops_sustained": d["bf16_tflops_sustained"],
                "hbm_gbs": d["hbm_gbs"], "source": "measured"}
    return {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0, "source": "fallback"}


# ----------------------------------------------------------------------------- dist plumbing
def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist

        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local) if backend == "nccl" else None)
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world: int) -> None:
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist

    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_teardown(world: int) -> None:
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and throttle-reason samples taken while the timed region runs.

    NVML is read from a thread every few milliseconds, so that a timed region of a tenth of a
    second still gets samples; ``nvidia-smi -lms`` is the fallback where NVML is unavailable.
    Only reads: no clock, power or other GPU setting is touched.
    """

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    PERIOD_S = 0.004

    def __init__(self, device: int):
        self.proc = None
        self.thread = None
        self.nvml = None
        self.samples = []  # (sm_mhz, set of reason names)
        self.sm_max = None
        try:
            props = torch.cuda.get_device_properties(device)
            self.gpu_id = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
        except Exception:
            self.gpu_id = str(device)
        try:
            import pynvml

            pynvml.nvmlInit()
            try:
                h = pynvml.nvmlDeviceGetHandleByPciBusId(self.gpu_id.upper())
            except Exception:
                h = pynvml.nvmlDeviceGetHandleByPciBusId(self.gpu_id)
            self.sm_max = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            self.bits = {"hw_slowdown": pynvml.nvmlClocksEventReasonHwSlowdown,
                         "hw_thermal_slowdown": pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                         "sw_thermal_slowdown": pynvml.nvmlClocksEventReasonSwThermalSlowdown,
                         "sw_power_cap": pynvml.nvmlClocksEventReasonSwPowerCap}
            self.nvml, self.handle = pynvml, h
        except Exception:
            self.nvml = None

    def _poll(self):
        n, h = self.nvml, self.handle
        while not self.stop_flag.is_set():
            try:
                mhz = float(n.nvmlDeviceGetClockInfo(h, n.NVML_CLOCK_SM))
                mask = n.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((mhz, {k for k, bit in self.bits.items() if mask & bit}))
            except Exception:
                pass
            self.stop_flag.wait(self.PERIOD_S)

    def start(self):
        if self.nvml is not None:
            self.stop_flag = threading.Event()
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            return
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.05)

    def stop(self) -> dict:
        if self.thread is not None:
            self.stop_flag.set()
            self.thread.join(timeout=5)
            sm = [mhz for mhz, _ in self.samples]
            reasons = set().union(*(r for _, r in self.samples)) if self.samples else set()
            return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.sm_max,
                    "samples": len(sm), "reasons": sorted(reasons), "source": "nvml"}
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "samples": 0, "reasons": ["clock sampling unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        sm, smax, reasons = [], [], set()
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(self.NAMES, parts[4:8]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "samples": len(sm), "reasons": sorted(reasons), "source": "nvidia-smi"}


def tensor_peak(peaks: dict, clk: dict) -> tuple[float, str]:
    """The measured bf16 peak for the clock regime the timed region ran in: the sustained
    figure (taken at ~1.3 GHz under the power cap) when the median sampled SM clock was below
    95 % of its maximum, else the burst figure (also when there are no samples: the larger
    denominator).  A power-cap flag seen at full clock is reported in `clocks` but did not
    lower the clock, so it does not switch the peak."""
    mhz, mx = clk.get("sm_mhz"), clk.get("sm_max_mhz")
    if mhz is not None and mx and mhz < 0.95 * mx:
        return peaks["bf16_tflops_sustained"], f"{peaks['source']} bf16 dense matmul, sustained (SM clock lowered)"
    why = "SM clock at its maximum" if mhz is not None else "no clock samples"
    return peaks["bf16_tflops"], f"{peaks['source']} bf16 dense matmul, burst ({why})"


def wait_event(ev, limit_s: float = 600.0) -> None:
    """Wait for a recorded CUDA event by polling with short sleeps, which release the GIL, so
    that the clock-sampling thread keeps running while the GPU works; give up with an error
    after limit_s seconds (the timed regions take well under a second)."""
    t0 = time.monotonic()
    while not ev.query():
        if time.monotonic() - t0 > limit_s:
            raise RuntimeError(f"timed region did not complete within {limit_s:.0f} s")
        time.sleep(0.0005)


# ----------------------------------------------------------------------------- end to end
def pipelined_e2e(h_in: dict, h_out: dict, make_set, compute, n_steps: int, world: int) -> dict:
    """Steps through the public API with host buffers, the way a caller streams them: every
    step copies its inputs in from pinned host memory and its results out to pinned host
    memory; the copy-in of step i+1 and the copy-out of step i-1 run on their own streams while
    step i's kernels run, on two sets of device buffers (events order the reuse of a set).
    ``make_set()`` -> (device inputs, device outputs) named like h_in / h_out;
    ``compute(dev_in, dev_out)`` enqueues one step on the current stream.  Returns the mean
    time per step over n_steps (max over ranks), copies included."""
    sets = [make_set() for _ in range(2)]
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    in_ready = [torch.cuda.Event() for _ in range(2)]
    cmp_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]

    def run(n):
        for i in range(n):
            b = i % 2
            din, dout = sets[b]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(cmp_done[b])  # step i-2 has finished reading this set's inputs
                for name, t in h_in.items():
                    din[name].copy_(t, non_blocking=True)
                in_ready[b].record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(in_ready[b])
                if i >= 2:
                    s_cmp.wait_event(out_done[b])  # step i-2's results have been copied out
                compute(din, dout)
                cmp_done[b].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(cmp_done[b])
                for name, t in h_out.items():
                    t.copy_(dout[name], non_blocking=True)
                out_done[b].record(s_out)

    run(2)  # warm-up (every buffer touched once)
    torch.cuda.synchronize()
    barrier(world)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    run(n_steps)
    t1.record(s_out)  # the last copy-out depends on every earlier copy and kernel
    torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1) / n_steps, world)
    return {"ms_per_step": ms, "steps": n_steps,
            "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in h_in.values()),
            "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in h_out.values()),
            "overlap": "copy-in of step i+1 and copy-out of step i-1 overlap step i (three streams, two "
                       "device buffer sets)"}


# ----------------------------------------------------------------------------- CPU oracle baseline
def oracle_head_step(inp_cpu: dict, w: inputs.Workload, b: int, h: int) -> None:
    import oracle

    g = h // (inp_cpu["q"].shape[1] // inp_cpu["k"].shape[1])  # key/value head (grouped-query runs)
    q, do = inp_cpu["q"][b, h], inp_cpu["do"][b, h]
    k, v = inp_cpu["k"][b, g], inp_cpu["v"][b, g]
    oracle.attention_forward(q, k, v, w.scale, w.causal)
    oracle.attention_backward(q, k, v, do, w.scale, w.causal)


def blas_threads() -> int:
    try:
        import threadpoolctl

        info = threadpoolctl.threadpool_info()
        return int(max(i.get("num_threads", 1) for i in info)) if info else 1
    except Exception:
        return len(os.sched_getaffinity(0))


def cpu_baseline(w: inputs.Workload, inp_cpu: dict, budget_s: float = 12.0) -> dict:
    """The oracle, as it stands, on whole heads of the workload until ~budget_s of CPU work.
    Sequences too long for the oracle's N x N matrices (N > 16384) are sampled the way their
    parity test checks them: the 4096-token causal prefix problem of a head, forward and
    backward."""
    import oracle

    P = 4096 if w.N > 16384 else w.N
    per_head = (w.fwd_flops + w.bwd_flops) / (w.B * w.H) * (P / w.N) ** 2
    heads, t0 = 0, time.perf_counter()
    while True:
        b, h = heads // w.H % w.B, heads % w.H
        if P == w.N:
            oracle_head_step(inp_cpu, w, b, h)
        else:
            q, k, v, do = (inp_cpu[n][b, h, :P] for n in ("q", "k", "v", "do"))
            oracle.attention_forward(q, k, v, w.scale, w.causal)
            oracle.attention_backward(q, k, v, do, w.scale, w.causal)
        heads += 1
        if time.perf_counter() - t0 > budget_s or heads >= w.B * w.H:
            break
    dt = time.perf_counter() - t0
    what = "heads" if P == w.N else f"heads' {P}-token prefix problems"
    return {"value": per_head * heads / dt / 1e12, "unit": "TFLOPS", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{heads} of {w.B * w.H} {what} (fwd+bwd, fp64 numpy, S and P materialised), {dt:.1f} s"}


def run_reference(args, rank: int, world: int) -> None:
    """--impl reference: the fp64 oracle timed on the host cores, one head per step."""
    if rank != 0:
        return
    w = inputs.workload(WORKLOAD)
    inp = inputs.make_inputs(w, device="cpu")
    per_head = (w.fwd_flops + w.bwd_flops) / (w.B * w.H)
    for i in range(args.warmup):
        oracle_head_step(inp, w, 0, i % w.H)
    t0 = time.perf_counter()
    for i in range(args.steps):
        oracle_head_step(inp, w, (i // w.H) % w.B, i % w.H)
    dt = time.perf_counter() - t0
    value = per_head * args.steps / dt / 1e12
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal,
                   "step": "one (b, h) head of the workload, forward + backward"},
        "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": cores, "kind": "oracle",
                         "sample": f"one head per step, {args.steps} steps"},
        "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- our arm
def run_ours(args, rank: int, world: int, local: int) -> None:
    from exact_io_aware_91_b200 import api

    w = inputs.workload(args.workload)
    if not w.backward:  # a forward-only workload (4): timed by the forward-only runner
        return run_fwd_only(args, rank, world, "plain")
    dev = torch.device("cuda", torch.cuda.current_device())
    B, H, N, d = w.B, w.H, w.N, w.d
    if args.head_dim == 256:  # the same B * H * d as the workload, with d = 256 (H halved)
        H, d = H * d // 256, 256
        w = inputs.Workload(f"causal_b{B}_h{H}_n{N}_d256" + ("_spiky" if w.spiky_frac else ""), B, H, N, d,
                            w.causal, w.dtype, w.dist, w.backward, w.spiky_frac, w.seed)
    Hkv = H if args.kv_heads is None else args.kv_heads
    if Hkv < 1 or H % Hkv:
        raise SystemExit(f"--kv-heads must divide H = {H}")
    name = w.name if Hkv == H else f"{w.name}_gqa_h{H}_hkv{Hkv}"
    window = (-1, -1) if args.window is None else (args.window, -1)
    if args.window is not None:
        name += f"_window{args.window}"
    # metric flops: 4 d per visible (query, key) pair and head forward, 2.5x that backward
    # (w.fwd_flops is the same count for the plain causal / full masks)
    if args.window is None:
        fwd_flops = w.fwd_flops
    else:
        pairs = 0
        for i in range(N):
            lo = max(0, i - args.window)
            hi = i if w.causal else N - 1
            pairs += hi - lo + 1
        fwd_flops = 4.0 * B * H * d * pairs
    bwd_flops = 2.5 * fwd_flops
    inp_cpu = inputs.make_qkv(B, H, N, d, dtype=w.dtype, dist=w.dist, spiky_frac=w.spiky_frac, backward=True,
                              seed=w.seed, kv_heads=None if Hkv == H else Hkv)
    q, k, v, do = (inp_cpu[n].to(dev) for n in ("q", "k", "v", "do"))
    o = torch.empty_like(q)
    res = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dq = torch.empty((B, H, N, d), dtype=torch.float32, device=dev)
    dk = torch.empty((B, Hkv, N, d), dtype=torch.float32, device=dev)
    dv = torch.empty_like(dk)
    ws_size = (api.fa_bwd_ws_workspace_size if args.window is None else api.fa_bwd_gqa_workspace_size)
    ws = torch.empty(ws_size(B, H, Hkv, N, d), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    # forward with a workspace: V converted to fp16 in one streaming pass, then the kernel
    fws = torch.empty(api.fa_fwd_workspace_size(B, Hkv, N, d), dtype=torch.uint8, device=dev)
    if args.window is None:
        def fwd_call(q, k, v, **kw):
            return api.fa_fwd_ws(q, k, v, workspace=fws, **kw)

        def bwd_call(q, k, v, o, do, lse, **kw):  # takes the forward's residual and its fp16 V copy
            return api.fa_bwd_ws(q, k, v, o, do, lse, fws, **kw)
    else:  # sliding window: the descriptor-based entry points
        def fwd_call(q, k, v, **kw):
            return api.fa_attn_fwd(q, k, v, window=window, workspace=fws, **kw)

        def bwd_call(*a, **kw):
            return api.fa_attn_bwd(*a, window=window, **kw)

    def step():
        fwd_call(q, k, v, causal=w.causal, scale=w.scale, o=o, lse=lse, o_resid=res)
        bwd_call(q, k, v, o, do, lse, causal=w.causal, scale=w.scale, workspace=ws, dq=dq, dk=dk, dv=dv,
                 o_resid=res)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if api.fa_last_device_status() != api.FA_OK:
        raise RuntimeError("device status not OK after warm-up")

    # ---- timed region: K steps, per-kernel events on the launching stream
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    clocks = ClockSampler(torch.cuda.current_device())
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for s in range(args.steps):
        e = ev[s]
        e[0].record(stream)
        fwd_call(q, k, v, causal=w.causal, scale=w.scale, o=o, lse=lse, o_resid=res)
        e[1].record(stream)
        api.fa_bwd_set_phase_events((e[2], e[3]))
        bwd_call(q, k, v, o, do, lse, causal=w.causal, scale=w.scale, workspace=ws, dq=dq, dk=dk, dv=dv,
                 o_resid=res)
        api.fa_bwd_set_phase_events(None)
        e[4].record(stream)
    end.record(stream)
    wait_event(end)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    total_ms = start.elapsed_time(end)
    total_ms_max = max_over_ranks(total_ms, world)
    if api.fa_last_device_status() != api.FA_OK:
        raise RuntimeError("device status not OK after the timed region")

    phase = {"fwd": [], "bwd_pre": [], "bwd_dkdv": [], "bwd_dq": []}
    for e in ev:
        phase["fwd"].append(e[0].elapsed_time(e[1]))
        phase["bwd_pre"].append(e[1].elapsed_time(e[2]))
        phase["bwd_dkdv"].append(e[2].elapsed_time(e[3]))
        phase["bwd_dq"].append(e[3].elapsed_time(e[4]))
    mean = {kk: statistics.mean(vv) for kk, vv in phase.items()}

    flops_step = fwd_flops + bwd_flops
    ms_step = total_ms_max / args.steps
    value = flops_step * world / (ms_step * 1e-3) / 1e12
    peaks = load_peaks()

    # dominant kernel (largest mean time) and its algorithmic flops per launch
    algo = {"fwd": fwd_flops,                  # QK^T and PV
            "bwd_dkdv": 2.0 * fwd_flops,        # K Q^T, V dO^T, P^T dO, dS^T Q (at d = 256 K Q^T runs in both kernels)
            "bwd_dq": 1.5 * fwd_flops}          # Q K^T, dO V^T, dS K
    dom = max(("fwd", "bwd_dkdv", "bwd_dq"), key=lambda kk: mean[kk])
    achieved = algo[dom] / (mean[dom] * 1e-3) / 1e12
    peak, peak_kind = tensor_peak(peaks, clk)
    roofline = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak,
                "traffic": args.traffic if args.traffic is not None else recorded_traffic(dom, name),
                "peak_kind": peak_kind}

    # ---- end to end through the public API with host buffers (pinned), copies inside the timed region
    e2e = None
    if not args.no_e2e:
        h_in = {n: inp_cpu[n].pin_memory() for n in ("q", "k", "v", "do")}
        h_out = {"o": torch.empty(o.shape, dtype=o.dtype).pin_memory(),
                 "lse": torch.empty(lse.shape, dtype=lse.dtype).pin_memory(),
                 "dq": torch.empty(dq.shape, dtype=dq.dtype).pin_memory(),
                 "dk": torch.empty(dk.shape, dtype=dk.dtype).pin_memory(),
                 "dv": torch.empty(dv.shape, dtype=dv.dtype).pin_memory()}

        def make_set():
            din = {n: torch.empty_like(t, device=dev) for n, t in h_in.items()}
            dout = {n: torch.empty_like(t, device=dev) for n, t in h_out.items()}
            dout["res"] = torch.empty_like(din["q"])  # the forward's residual, used by the backward
            return din, dout

        def compute(din, dout):
            fwd_call(din["q"], din["k"], din["v"], causal=w.causal, scale=w.scale, o=dout["o"], lse=dout["lse"],
                     o_resid=dout["res"])
            bwd_call(din["q"], din["k"], din["v"], dout["o"], din["do"], dout["lse"], causal=w.causal,
                     scale=w.scale, workspace=ws, dq=dout["dq"], dk=dout["dk"], dv=dout["dv"], o_resid=dout["res"])

        e2e = pipelined_e2e(h_in, h_out, make_set, compute, max(4, min(args.steps, 8)), world)
        e2e = {"value": flops_step * world / (e2e["ms_per_step"] * 1e-3) / 1e12, "unit": "TFLOPS", **e2e}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.window is None:
        cpu = cpu_baseline(w, inp_cpu)  # (the oracle timing covers the unwindowed problem)

    if rank == 0:
        # the headline metric names workload 3 (N = 8192, d = 128); other shapes say what they are
        metric = (METRIC if (args.workload == WORKLOAD and d == 128) else
                  f"attention fwd/bwd TFLOPS (BF16, {'causal' if w.causal else 'non-causal'}, N={N}, d={d})")
        line = {
            "metric": metric, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": name, "B": B, "H": H, "H_kv": Hkv, "N": N, "d": d, "causal": w.causal,
                       "window": list(window),
                       "global_batch": B * world, "seq_len": N, "parallelism": f"replicas{world}",
                       "l2": (f"inputs larger than L2 (Q, K, V, dO, O {B * H * N * d * 2 / 1e6:.0f} MB each > 126 MB)"
                              if B * H * N * d * 2 > 126e6 else "small workload: inputs may stay in L2")},
            "fwd_tflops": fwd_flops / (mean["fwd"] * 1e-3) / 1e12,
            "bwd_tflops": bwd_flops / ((mean["bwd_pre"] + mean["bwd_dkdv"] + mean["bwd_dq"]) * 1e-3) / 1e12,
            # the products the separate dK/dV and dQ kernels execute: 3.5x the forward's flops
            # (S and dP are formed in both; at d = 256 4x: S^T also in both the dV and the dK
            # kernel), against the metric's 2.5x
            "bwd_executed_tflops": (4.0 if d == 256 else 3.5) * fwd_flops
                                   / ((mean["bwd_pre"] + mean["bwd_dkdv"] + mean["bwd_dq"]) * 1e-3) / 1e12,
            "kernel_ms": mean,
            "frac_of_peak": {"measured_burst": value / world / peaks["bf16_tflops"],
                             "measured_sustained": value / world / peaks["bf16_tflops_sustained"],
                             "datasheet_2250": value / world / 2250.0},
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": e2e,
            # V pass + its fix-up + forward, preprocess + its fix-up, dK/dV (two kernels at d = 256),
            # dQ; plus the partial-sum reduce when the library splits a group's query heads (fewer
            # than 4 x 148 dK/dV units)
            "gpu_launches": args.steps * (7 + (1 if d == 256 else 0)
                                          + (1 if H // Hkv > 1 and B * Hkv * ((N + 127) // 128) < 592 else 0)),
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- forward-only runs
METRIC_FP8 = "attention fwd TFLOPS (FP8 E4M3 inputs, causal, N=8k, d=128) & % of B200 fp8 tensor peak"
METRIC_D256 = "attention fwd TFLOPS (BF16, causal, N=8k, d=256) & % of B200 tensor peak"


def run_fwd_only(args, rank: int, world: int, kind: str) -> None:
    """--fp8: the 8-bit forward (fa_attn_fwd_fp8) on the workload's shape (3 by default; 4 for d = 64).  --head-dim 256: the
    bf16 forward with d = 256 (fa_fwd_ws) on B = 2, H = 16, N = 8192 (workload 3's B * H * d).
    kind "plain": a forward-only workload (4) on its own shape, whose roofline is the larger
    of its HBM time and its tensor-core time.  Forward only; L2 flushed between the timed
    forwards."""
    from exact_io_aware_91_b200 import api

    w = inputs.workload(args.workload)
    fp8, plain = kind == "fp8", kind == "plain"
    if fp8 or plain:
        B, H, N, d = w.B, w.H, w.N, w.d
    else:
        B, H, N, d = w.B, w.H * w.d // 256, w.N, 256
    scale = 1.0 / 16.0 if kind == "d256" else w.scale
    fwd_flops = 4.0 * B * H * N * N * d / (2 if w.causal else 1)
    # algorithmic bytes: Q, K, V read and O written in bf16 (8-bit inputs: one byte each), LSE
    fwd_bytes = (3 * (1 if fp8 else 2) + 2) * B * H * N * d + 4 * B * H * N
    if fp8:
        x = inputs.make_qkv_fp8(B, H, N, d, dist=w.dist, spiky_frac=w.spiky_frac, seed=w.seed + rank)
        host_in = {n: x[n].view(torch.uint8) for n in ("q", "k", "v")}
    else:
        x = inputs.make_qkv(B, H, N, d, dtype=torch.bfloat16, dist=w.dist, spiky_frac=w.spiky_frac,
                            backward=False, seed=w.seed + rank)
        host_in = {n: x[n] for n in ("q", "k", "v")}
    dev_in = {n: t.cuda() for n, t in host_in.items()}
    o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    pr = api.FaAttnProblem(B, H, H, N, d, scale, int(w.causal), -1, -1)
    ws_bytes = api.fa_attn_fwd_fp8_workspace_size(pr) if fp8 else api.fa_attn_fwd_workspace_size(pr)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")  # > the 126 MB L2
    stream = torch.cuda.current_stream()

    def compute(din, dout):
        if fp8:
            api.fa_attn_fwd_fp8(din["q"].view(torch.float8_e4m3fn), din["k"].view(torch.float8_e4m3fn),
                                din["v"].view(torch.float8_e4m3fn), x["q_descale"], x["k_descale"], x["v_descale"],
                                causal=w.causal, scale=pr.scale, o=dout["o"], lse=dout["lse"], workspace=ws)
        else:
            api.fa_fwd_ws(din["q"], din["k"], din["v"], causal=w.causal, scale=pr.scale, o=dout["o"],
                          lse=dout["lse"], workspace=ws)

    dev_out = {"o": o, "lse": lse}
    for _ in range(args.warmup):
        compute(dev_in, dev_out)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    clocks = ClockSampler(torch.cuda.current_device())
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    for e0, e1 in ev:
        flush.zero_()  # L2 flushed between timed forwards (outside the events)
        e0.record(stream)
        compute(dev_in, dev_out)
        e1.record(stream)
    wait_event(ev[-1][1])
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    if api.fa_last_device_status() != api.FA_OK:
        raise RuntimeError("device status not OK after the timed region")
    ms = [a.elapsed_time(b) for a, b in ev]
    ms_step = max_over_ranks(sum(ms), world) / args.steps
    value = fwd_flops * world / (ms_step * 1e-3) / 1e12
    peaks = load_peaks()
    bf16_peak, peak_kind = tensor_peak(peaks, clk)
    ratio = 2.0 if fp8 else 1.0  # dense fp8 = 2x dense bf16 (4.5 vs 2.25 PFLOP/s nominal)
    mean_s = statistics.mean(ms) * 1e-3
    achieved = fwd_flops / mean_s / 1e12
    achieved_gbs = fwd_bytes / mean_s / 1e9
    name = (w.name + "_fp8" if fp8 else w.name if plain else f"causal_b{B}_h{H}_n{N}_d256_spiky")
    dom = "fwd_fp8" if fp8 else "fwd" if plain else "fwd_d256"
    traffic = args.traffic if args.traffic is not None else recorded_traffic(dom, name)
    # the bound: HBM when moving the algorithmic bytes at the measured copy bandwidth takes longer
    # than the products at the tensor peak
    hbm_bound = fwd_bytes / (peaks["hbm_gbs"] * 1e9) > fwd_flops / (ratio * bf16_peak * 1e12)
    if hbm_bound:
        roofline = {"bound": "hbm", "kernel": dom, "achieved": achieved_gbs, "peak": peaks["hbm_gbs"],
                    "unit": "GB/s", "frac": achieved_gbs / peaks["hbm_gbs"], "traffic": traffic,
                    "peak_kind": f"{peaks['source']} copy bandwidth"}
    else:
        roofline = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": ratio * bf16_peak,
                    "unit": "TFLOP/s", "frac": achieved / (ratio * bf16_peak), "traffic": traffic,
                    "peak_kind": peak_kind.replace("bf16 dense matmul",
                                                   "bf16 dense matmul x 2 (fp8 / bf16 nominal ratio)" if fp8
                                                   else "bf16 dense matmul")}

    e2e = None
    if not args.no_e2e:
        h_in = {n: t.pin_memory() for n, t in host_in.items()}
        h_out = {"o": torch.empty(o.shape, dtype=o.dtype).pin_memory(),
                 "lse": torch.empty(lse.shape, dtype=lse.dtype).pin_memory()}

        def make_set():
            return ({n: torch.empty_like(t, device="cuda") for n, t in h_in.items()},
                    {n: torch.empty_like(t, device="cuda") for n, t in h_out.items()})

        e2e = pipelined_e2e(h_in, h_out, make_set, compute, max(4, min(args.steps, 8)), world)
        e2e = {"value": fwd_flops * world / (e2e["ms_per_step"] * 1e-3) / 1e12, "unit": "TFLOPS", **e2e}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle

        per_head = fwd_flops / (B * H)
        heads, t0 = 0, time.perf_counter()
        codes = {n: t.numpy() for n, t in host_in.items()} if fp8 else None
        while True:
            b, h = heads // H % B, heads % H
            if fp8:
                oracle.attention_forward_fp8(codes["q"][b:b + 1, h:h + 1], codes["k"][b:b + 1, h:h + 1],
                                             codes["v"][b:b + 1, h:h + 1], x["q_descale"], x["k_descale"],
                                             x["v_descale"], scale, w.causal)
            else:
                oracle.attention_forward(x["q"][b, h], x["k"][b, h], x["v"][b, h], scale, w.causal)
            heads += 1
            if time.perf_counter() - t0 > 12.0 or heads >= B * H:
                break
        dt = time.perf_counter() - t0
        what = "forward of the dequantized E4M3 inputs" if fp8 else f"forward, d = {d}"
        cpu = {"value": per_head * heads / dt / 1e12, "unit": "TFLOPS", "cores": blas_threads(), "kind": "oracle",
               "sample": f"{heads} of {B * H} heads ({what}, fp64 numpy), {dt:.1f} s"}

    if rank == 0:
        line = {
            "metric": (METRIC_FP8 if fp8 and args.workload == WORKLOAD else
                       f"attention fwd TFLOPS (FP8 E4M3 inputs, {'causal' if w.causal else 'non-causal'}, N={N}, "
                       f"d={d})" if fp8 else METRIC_D256 if not plain else
                       f"attention fwd TFLOPS (BF16, {'causal' if w.causal else 'non-causal'}, N={N}, d={d})"),
            "value": value, "unit": "TFLOPS", "n_gpus": world, "achieved_gbs": achieved_gbs,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "e4m3" if fp8 else "bf16", "data": "synthetic",
            "config": {"workload": name, "B": B, "H": H, "N": N, "d": d, "causal": w.causal,
                       "global_batch": B * world, "seq_len": N, "parallelism": f"replicas{world}",
                       "step": "forward only", "l2": "flushed between timed forwards (256 MB write)"},
            "frac_of_peak": {"measured_burst": value / world / (ratio * peaks["bf16_tflops"]),
                             "measured_sustained": value / world / (ratio * peaks["bf16_tflops_sustained"]),
                             "datasheet": value / world / (ratio * 2250.0)},
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": e2e,
            # the persistent forward per step (the 8-bit one's work counter is reset by a memset;
            # the bf16 ones follow the V pass and its fix-up)
            "gpu_launches": args.steps * (1 if fp8 else 3),
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", type=int, default=WORKLOAD, choices=[2, 3, 4, 5],
                    help="workload index (3 = the metric's; others for profiling runs)")
    ap.add_argument("--kv-heads", type=int, default=None,
                    help="grouped-query run: K/V with this many heads (fa_fwd_ws / fa_bwd_ws); default H")
    ap.add_argument("--window", type=int, default=None,
                    help="sliding-window run: each query sees the previous WINDOW keys and itself "
                         "(fa_attn_fwd / fa_attn_bwd); default no window")
    ap.add_argument("--head-dim", type=int, default=None, choices=[256],
                    help="head dimension 256 on the workload's B * H * d (B=2, H=16, N=8192): forward + "
                         "backward (fa_fwd_ws, fa_bwd_ws); with --fwd-only the forward alone")
    ap.add_argument("--fwd-only", action="store_true", help="with --head-dim 256: time the forward alone")
    ap.add_argument("--fp8", action="store_true",
                    help="time the 8-bit forward (E4M3 inputs, fa_attn_fwd_fp8) on the workload's shape")
    ap.add_argument("--traffic", type=float, default=None,
                    help="DRAM bytes per launch of the dominant kernel from an ncu capture (reported as-is)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank, world, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        elif args.fp8:
            run_fwd_only(args, rank, world, "fp8")
        elif args.head_dim == 256 and args.fwd_only:
            run_fwd_only(args, rank, world, "d256")
        else:
            run_ours(args, rank, world, local)
    finally:
        dist_teardown(world)


if __name__ == "__main__":
    main()
