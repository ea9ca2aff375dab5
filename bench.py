#!/usr/bin/env python
"""Benchmark of the SSD mixer forward (conv1d+SiLU then chunked selective scan).

One step = the whole layer over one batch of the workload: by default the
Video-Ma2mba-0.3B mixer shape (32 heads, P=64, N=128, Q=128, bf16) over a
1,048,576-token stream processed as 8 consecutive 131072-token segments, each
resumed from the previous segment's (state, conv tail), with state
checkpoints every 4096 tokens.  Inputs are seeded synthetic tensors already
resident in HBM (u alone is 4.8 GB, far larger than the 126 MB L2).

Prints ONE JSON line (rank 0).  Multi-GPU: `torchrun --nproc-per-node N
bench.py --gpus N`; every rank runs its own independent stream (weak
scaling, no data-path collective), NCCL only for the barrier and the
max-over-ranks time.  `--impl reference` times the CPU oracle instead.
"""
import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import ssd_synth  # noqa: E402

METRIC = "SSD mixer fwd tokens/s at 0.3B shape, L=1M; % of HBM/tensor roofline"
DEFAULT_WORKLOAD = "mamba2-0.3b-L1M-stream8"
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(ssd_synth.BY_NAME))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample-tokens", type=int, default=393216)
    # profiling aids: run a shorter stream of the same shape (not a bench line)
    ap.add_argument("--seq-len", type=int, default=None)
    ap.add_argument("--segments", type=int, default=None)
    # the decode step instead of the headline step: this many independent streams of the
    # 0.3B shape, each advancing one token per step (its own JSON line)
    ap.add_argument("--decode-streams", type=int, default=0)
    # the backward pass of the scan instead of the headline step: gradients from the
    # forward's checkpoints, on the 0.3B 16384-token workload (its own JSON line)
    ap.add_argument("--backward", action="store_true")
    # the backward pass of the whole layer (conv1d + SiLU, then the scan) from the forward's state
    # checkpoints and conv buffers, on the same workload (its own JSON line)
    ap.add_argument("--layer-backward", action="store_true")
    # the gated RMS norm of the layer output on one 131072-token segment of the 0.3B shape
    ap.add_argument("--gated-norm", action="store_true")
    # the layer as two library calls (conv over every channel, then the scan) instead of the
    # default one call, whose first scan pass computes the conv of x itself
    ap.add_argument("--two-call", action="store_true")
    return ap.parse_args()


# ----------------------------------------------------------------- bytes model
def algorithmic_bytes_per_token(wl):
    """Minimum HBM bytes per token of the two-call path (conv, then scan)."""
    e = 2 if wl.dtype == "bf16" else 4
    conv = 2 * wl.cch * e                              # read u, write v
    scan = (2 * wl.d_inner * e                         # read x, write y
            + 2 * wl.G * wl.N * e                      # read B, C
            + 4 * wl.H                                 # read dt
            + (4 * wl.H * wl.P * wl.N / wl.s if wl.s else 0))  # write checkpoints
    return conv, scan


def layer_bytes_per_token(wl):
    """Minimum HBM bytes per token of the layer itself: read u and dt, write y and the
    checkpoints (the conv output need not leave the chip)."""
    e = 2 if wl.dtype == "bf16" else 4
    return (wl.cch * e + 4 * wl.H + wl.d_inner * e
            + (4 * wl.H * wl.P * wl.N / wl.s if wl.s else 0))


def issued_mma_flops_per_token(wl):
    """Dense bf16 MMA flops the tensor-core output pass issues per token (per chunk of Q
    tokens and head pair: G = C B^T, Ys = C hp^T, S = B^T (w o X), each Q x 128 x N (or
    x Q), and Y = Pm X for both heads, Q x P x Q each)."""
    per_pair_chunk = 2 * (wl.Q * 128 * wl.N * 2 + 128 * wl.N * wl.Q + 2 * wl.Q * wl.P * wl.Q)
    return per_pair_chunk * (wl.H // 2) / wl.Q


def bf16_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


# ----------------------------------------------------------------- peaks
def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def recorded_traffic(kernel):
    """DRAM bytes per token of `kernel` from the committed ncu summary, or None
    when the kernel's source changed since those counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        rec = d[kernel]
        src = os.path.join(ROOT, rec["source"])
        digest = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        if digest != rec["source_sha256_16"]:
            return None
        return float(rec["dram_bytes_per_token"])
    except Exception:
        return None


# ----------------------------------------------------------------- clocks
class NvmlClockSampler:
    """SM clock, power and throttle reasons every 2 ms from a thread (NVML), so that
    timed regions of a few milliseconds are still sampled while they run."""

    def __init__(self, device_index):
        import threading
        import pynvml
        self.nv = pynvml
        pynvml.nvmlInit()
        # NVML numbers the physical GPUs; find this process's CUDA device by its PCI address
        prop = torch.cuda.get_device_properties(device_index)
        bus = "%08X:%02X:%02X.0" % (prop.pci_domain_id, prop.pci_bus_id, prop.pci_device_id)
        try:
            self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except pynvml.NVMLError:
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
        self.rows = []
        self.stop_flag = threading.Event()
        self.thread = threading.Thread(target=self._run, daemon=True)

    def _sample(self):
        nv = self.nv
        r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        self.rows.append({"sm": nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM),
                          "max": nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM),
                          "power": nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0, "bits": r})

    def _run(self):
        while not self.stop_flag.is_set():
            self._sample()
            time.sleep(0.002)

    def start(self):
        self._sample()
        self.thread.start()

    def stop(self):
        self.stop_flag.set()
        self.thread.join(timeout=5)
        self._sample()
        rows = self.rows[1:-1] or self.rows
        nv = self.nv
        names = ((nv.nvmlClocksEventReasonHwSlowdown, "hw_slowdown"),
                 (nv.nvmlClocksEventReasonHwThermalSlowdown, "hw_thermal_slowdown"),
                 (nv.nvmlClocksEventReasonSwThermalSlowdown, "sw_thermal_slowdown"),
                 (nv.nvmlClocksEventReasonSwPowerCap, "sw_power_cap"))
        reasons = sorted({name for r in rows for bit, name in names if r["bits"] & bit})
        loaded = [r for r in rows if r["power"] > 200] or rows
        return {"sm_mhz": statistics.median(r["sm"] for r in loaded), "sm_max_mhz": max(r["max"] for r in rows),
                "reasons": reasons, "samples": len(rows), "samples_under_load": len(loaded), "source": "nvml"}


def clock_sampler(device_index):
    try:
        return NvmlClockSampler(device_index)
    except Exception:
        return ClockSampler(device_index)


class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append({"sm": float(parts[1]), "max": float(parts[2]), "power": float(parts[3]),
                             "hw": parts[5], "hw_thermal": parts[6], "sw_thermal": parts[7],
                             "sw_power": parts[8]})
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        loaded = [r for r in rows if r["power"] > 200] or rows
        reasons = set()
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hw_thermal", "hw_thermal_slowdown"),
                              ("sw_thermal", "sw_thermal_slowdown"), ("sw_power", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in loaded),
                "sm_max_mhz": max(r["max"] for r in rows), "reasons": sorted(reasons),
                "samples": len(rows), "samples_under_load": len(loaded)}


# ----------------------------------------------------------------- distributed
def dist_setup(backend=None):
    """One process per GPU (RANK/LOCAL_RANK/WORLD_SIZE from torchrun).  NCCL on
    GPUs; gloo when no GPU is present (the CPU tests of the multi-rank logic)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if backend is None:
        backend = "nccl" if torch.cuda.is_available() else "gloo"
    if world > 1:
        import datetime
        import torch.distributed as dist
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def _nccl():
    import torch.distributed as dist
    return dist.is_initialized() and dist.get_backend() == "nccl"


def barrier(world, local):
    if world > 1:
        import torch.distributed as dist
        if _nccl():
            dist.barrier(device_ids=[local])
        else:
            dist.barrier()


def max_over_ranks(world, value):
    """Max of a per-rank scalar (the device time of the timed region)."""
    if world == 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device="cuda" if _nccl() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(wl, rank):
    """Every rank runs its own independent sequence (weak scaling)."""
    return wl.seed + 100 * rank


def job_throughput(wl, world, steps, ms_max):
    """Tokens of all ranks over the slowest rank's time."""
    return wl.tokens * world * steps / (ms_max / 1e3)


# ----------------------------------------------------------------- the workload
class Layer:
    """Device buffers and one step of the layer for a workload (one rank)."""

    def __init__(self, wl, seed, fused=True):
        import mamba_selective_state_causal_b200 as ssd
        self.ssd = ssd
        self.wl = wl
        self.fused = fused
        self.two_call = not fused
        d = torch.device("cuda", torch.cuda.current_device())
        self.dev = d
        prm = ssd_synth.make_params(wl, device=d, seed=seed)
        self.w, self.bias, self.A, self.D = prm["w"], prm["bias"], prm["A"], prm["D"]
        self.u = ssd_synth.make_u(wl, device=d, seed=seed)
        self.dt = ssd_synth.make_dt(wl, prm["dt_bias"], device=d, seed=seed)
        # inputs smaller than twice the L2 are rotated over copies at other addresses, so that
        # no step reads inputs the previous step left in L2
        l2 = getattr(torch.cuda.get_device_properties(d), "L2_cache_size", 126 * 2 ** 20) or 126 * 2 ** 20
        in_bytes = self.u.numel() * self.u.element_size() + self.dt.numel() * 4
        self.sets = [(self.u, self.dt)] + [(self.u.clone(), self.dt.clone())
                                           for _ in range(max(1, math.ceil(2 * l2 / in_bytes)) - 1)]
        self.cur = 0
        self.l2_note = ("inputs larger than L2 (u alone %.1f GB)" % (self.u.numel() * 2 / 1e9)
                        if len(self.sets) == 1 else
                        "inputs rotated over %d copies, %.2f GB in all, more than twice the %d MB L2"
                        % (len(self.sets), len(self.sets) * in_bytes / 1e9, l2 // 2 ** 20))
        seg = wl.seg_len
        self.seg = seg
        tdt = ssd_synth.torch_dtype(wl.dtype)
        self.v = None if fused else torch.empty(wl.b, seg, wl.cch, dtype=tdt, device=d)
        self.y = torch.empty(wl.b, wl.L, wl.H, wl.P, dtype=tdt, device=d)
        self.h = torch.empty(wl.b, wl.H, wl.P, wl.N, dtype=torch.float32, device=d)
        self.tail = torch.empty(wl.b, 3, wl.cch, dtype=tdt, device=d)
        n_ck = seg // wl.s if wl.s else 0
        self.ckpt = torch.empty(wl.b, wl.segments * n_ck, wl.H, wl.P, wl.N, dtype=torch.float32, device=d)
        if fused:
            code = ssd.SSD_BF16 if wl.dtype == "bf16" else ssd.SSD_F32
            self.ws = torch.empty(max(1, ssd.stream_workspace_size(wl.b, seg, wl.H, wl.P, wl.N, wl.G, wl.Q, code)),
                                  dtype=torch.uint8, device=d)
        else:
            self.ws = ssd.alloc_workspace(wl.b, seg, wl.H, wl.P, wl.N, wl.Q, d)
        self.n_ck = n_ck

    def segment(self, k, stream=None):
        wl, ssd = self.wl, self.ssd
        t0, t1 = k * self.seg, (k + 1) * self.seg
        u, dt = self.sets[self.cur]
        if self.two_call:
            # the conv over every channel, then the scan on its output: two library calls
            di, gn = wl.H * wl.P, wl.G * wl.N
            ssd.conv_forward(u[:, t0:t1], self.w, self.bias, tail_in=None if k == 0 else self.tail,
                             tail_out=self.tail, v=self.v, stream=stream)
            ssd.scan_forward(self.v[:, :, :di], self.v[:, :, di:di + gn], self.v[:, :, di + gn:],
                             dt[:, t0:t1], self.A, self.D, None if k == 0 else self.h, H=wl.H, G=wl.G,
                             Q=wl.Q, s=wl.s, y=self.y[:, t0:t1], h_final=self.h,
                             h_ckpt=self.ckpt[:, k * self.n_ck:(k + 1) * self.n_ck] if self.n_ck else None,
                             workspace=self.ws, stream=stream)
            return
        ssd.stream_forward(
            u[:, t0:t1], self.w, dt[:, t0:t1], self.A, self.D, H=wl.H, P=wl.P, N=wl.N,
            G=wl.G, Q=wl.Q, s=wl.s, conv_bias=self.bias,
            tail_in=None if k == 0 else self.tail, tail_out=self.tail,
            h0=None if k == 0 else self.h, h_final=self.h, v=self.v, y=self.y[:, t0:t1],
            h_ckpt=self.ckpt[:, k * self.n_ck:(k + 1) * self.n_ck] if self.n_ck else None,
            workspace=self.ws, stream=stream, keep_v=not self.fused)

    def step(self, stream=None):
        self.cur = (self.cur + 1) % len(self.sets)
        for k in range(self.wl.segments):
            self.segment(k, stream)


def time_steps(fn, steps, warmup, world, local):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    barrier(world, local)
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(steps):
        fn()
    e1.record(st)
    torch.cuda.synchronize()
    barrier(world, local)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def cpu_baseline(wl, sample_tokens):
    """The CPU oracle (as it stands) on a bounded sample of the same workload."""
    import oracle
    sw = ssd_synth.scaled(wl, L=sample_tokens, b=1, segments=1)
    prm = ssd_synth.make_params(sw)
    u = ssd_synth.make_u(sw).float().numpy()
    dt = ssd_synth.make_dt(sw, prm["dt_bias"]).numpy()
    args = (u, prm["w"].numpy(), dt, prm["A"].numpy(), prm["D"].numpy(), prm["bias"].numpy())
    t0 = time.perf_counter()
    oracle.layer(*args, None, None, H=sw.H, P=sw.P, N=sw.N, G=sw.G, s=sw.s,
                 io_round="bf16" if sw.dtype == "bf16" else "f32", want_ckpt=True)
    el = time.perf_counter() - t0
    return {"value": sample_tokens / el, "unit": "tokens/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{wl.name} shape, first {sample_tokens} tokens of one sequence, all {wl.H} heads, "
                      f"conv1d+SiLU then the per-token recurrence in fp64 ({el:.1f} s)"}


def run_reference(args, wl, world, rank):
    """--impl reference: the CPU oracle timed per step on a bounded sample."""
    if rank != 0:
        return
    import oracle
    sample = min(16384, wl.seg_len)
    sw = ssd_synth.scaled(wl, L=sample, b=1, segments=1)
    prm = ssd_synth.make_params(sw)
    u = ssd_synth.make_u(sw).float().numpy()
    dt = ssd_synth.make_dt(sw, prm["dt_bias"]).numpy()

    def step():
        oracle.layer(u, prm["w"].numpy(), dt, prm["A"].numpy(), prm["D"].numpy(), prm["bias"].numpy(),
                     None, None, H=sw.H, P=sw.P, N=sw.N, G=sw.G, s=sw.s, io_round="bf16")
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    value = sample * args.steps / el
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * el / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "sample_tokens_per_step": sample},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.num_threads(),
                         "kind": "oracle",
                         "sample": f"{wl.name} shape, {sample} tokens of one sequence per step, all heads"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_e2e(layer, steps=3):
    """Same metric through the library with host buffers: every step copies the
    inputs in from pinned host memory and the outputs back (y, the checkpoints and
    h_final).  Copies in, compute and copies out run on three streams, as a caller
    streaming a long input would run them, with dependencies per segment: a
    segment's input copy waits only for the previous step's compute of that
    segment (its slice of the device input), and a segment's compute for the
    previous step's output copy of that segment (its slices of y and of the
    checkpoints; the last segment's copy also holds h_final, which segment 0
    rewrites)."""
    wl = layer.wl
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    h_u = torch.empty(layer.u.shape, dtype=layer.u.dtype, pin_memory=True)
    h_dt = torch.empty(layer.dt.shape, dtype=layer.dt.dtype, pin_memory=True)
    h_u.copy_(layer.u)
    h_dt.copy_(layer.dt)
    o_y = torch.empty(layer.y.shape, dtype=layer.y.dtype, pin_memory=True)
    o_h = torch.empty(layer.h.shape, dtype=layer.h.dtype, pin_memory=True)
    o_ck = torch.empty(layer.ckpt.shape, dtype=layer.ckpt.dtype, pin_memory=True)
    seg, nseg, nck = layer.seg, wl.segments, layer.n_ck

    layer.cur = 0                     # the host copies land in the first input set
    prev_comp = [None] * nseg         # the previous step's compute of each segment
    prev_out = [None] * nseg          # the previous step's output copy of each segment

    def step():
        landed = []
        for k in range(nseg):
            t0, t1 = k * seg, (k + 1) * seg
            if prev_comp[k] is not None:
                s_in.wait_event(prev_comp[k])
            with torch.cuda.stream(s_in):
                layer.u[:, t0:t1].copy_(h_u[:, t0:t1], non_blocking=True)
                layer.dt[:, t0:t1].copy_(h_dt[:, t0:t1], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(s_in)
                landed.append(ev)
        for k in range(nseg):
            t0, t1 = k * seg, (k + 1) * seg
            comp.wait_event(landed[k])
            if prev_out[k] is not None:
                comp.wait_event(prev_out[k])
            if k == 0 and prev_out[nseg - 1] is not None:
                comp.wait_event(prev_out[nseg - 1])   # h_final of the previous step is out
            layer.segment(k, comp)
            done = torch.cuda.Event()
            done.record(comp)
            prev_comp[k] = done
            s_out.wait_event(done)
            with torch.cuda.stream(s_out):
                o_y[:, t0:t1].copy_(layer.y[:, t0:t1], non_blocking=True)
                if nck:
                    o_ck[:, k * nck:(k + 1) * nck].copy_(layer.ckpt[:, k * nck:(k + 1) * nck], non_blocking=True)
                if k == nseg - 1:
                    o_h.copy_(layer.h, non_blocking=True)
                out = torch.cuda.Event()
                out.record(s_out)
                prev_out[k] = out
    step()
    comp.wait_stream(s_out)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    for _ in range(steps):
        step()
    comp.wait_stream(s_out)           # every step's results are on the host
    e1.record(comp)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    h2d = h_u.numel() * h_u.element_size() + h_dt.numel() * h_dt.element_size()
    d2h = sum(t.numel() * t.element_size() for t in (o_y, o_h, o_ck))
    return {"value": wl.tokens / (ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ms, "steps": steps,
            "overlap": "copies in, compute and copies out on three streams, ordered per segment"}


def run_decode(args, world, rank, local):
    """Decode steps: each of B independent streams of the 0.3B shape takes one token per step
    (conv tail and state updated in place), timed with CUDA events like the headline step."""
    import __graft_entry__
    __graft_entry__.build()
    import mamba_selective_state_causal_b200 as ssd
    nb = args.decode_streams
    base = ssd_synth.BY_NAME[DEFAULT_WORKLOAD]
    n_tok = args.warmup + args.steps
    wl = ssd_synth.scaled(base, b=nb, L=n_tok, segments=1, name=f"decode-0.3b-{nb}streams")
    d = torch.device("cuda", torch.cuda.current_device())
    seed = rank_seed(wl, rank)
    prm = ssd_synth.make_params(wl, device=d, seed=seed)
    u_steps = ssd_synth.make_u(wl, device=d, seed=seed).transpose(0, 1).contiguous()     # [T][B][C_ch]
    dt_steps = ssd_synth.make_dt(wl, prm["dt_bias"], device=d, seed=seed).transpose(0, 1).contiguous()
    h = torch.zeros(nb, wl.H, wl.P, wl.N, dtype=torch.float32, device=d)
    tail = torch.zeros(nb, 3, wl.cch, dtype=u_steps.dtype, device=d)
    y = torch.empty(nb, wl.H, wl.P, dtype=u_steps.dtype, device=d)
    t = [0]

    def step():
        ssd.decode_step(u_steps[t[0]], prm["w"], dt_steps[t[0]], prm["A"], prm["D"], H=wl.H, P=wl.P,
                        N=wl.N, G=wl.G, conv_bias=prm["bias"], tail_in=tail, tail_out=tail,
                        h_in=h, h_out=h, y=y)
        t[0] += 1

    clocks = clock_sampler(local)
    clocks.start()
    ms = time_steps(step, args.steps, args.warmup, world, local)
    clk = clocks.stop()
    ssd.sync_status()
    ms = max_over_ranks(world, ms)
    e = 2
    step_bytes = nb * (2 * 4 * wl.H * wl.P * wl.N          # state read + write
                       + e * wl.cch + 2 * e * 3 * wl.cch     # token in, conv tail read + write
                       + e * wl.H * wl.P + 4 * wl.H)         # y out, dt in
    peak, peak_src = hbm_peak()
    achieved = step_bytes / (ms / args.steps / 1e3) / 1e9
    line = {
        "metric": "SSD decode step tokens/s (independent streams of the 0.3B shape)",
        "value": nb * world * args.steps / (ms / 1e3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": wl.name, "streams": nb, "heads": wl.H, "headdim": wl.P, "d_state": wl.N,
                   "l2": "state larger than L2 (%.0f MB)" % (nb * wl.H * wl.P * wl.N * 4 / 1e6)
                   if nb * wl.H * wl.P * wl.N * 4 > 126e6 else "state fits in L2"},
        "roofline": {"bound": "hbm", "kernel": "decode_step", "achieved": achieved, "peak": peak,
                     "unit": "GB/s", "frac": achieved / peak, "peak_source": peak_src, "traffic": None,
                     "algorithmic_bytes_per_launch": step_bytes},
        "gpu_launches": 2 * args.steps,
        "clocks": clk,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


# fp32 FMA issue of the CUDA cores: 148 SMs x 128 lanes x 2 flops x 1.965 GHz (max SM clock)
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def bwd_flops_per_chunk_head(P, N, Q=64):
    """Multiply-add flops of one (64-token chunk, head) in the backward kernels:
    summaries S and Gl (2 x 2QPN); gradients: C.B and dy.x (2Q^2 N + 2Q^2 P),
    dx (2Q^2 P + 2QNP), dB (2Q^2 N + 2QPN), dC (2QPN + 2Q^2 N)."""
    summary = 2 * 2 * Q * P * N
    grad = Q * Q * (6 * N + 4 * P) + 6 * Q * P * N
    return summary, grad


def bwd_grad_bytes_per_chunk_head(wl, Q=64):
    """Bytes one (64-token chunk, head) of the gradient kernel must move: read x and dy, the
    chunk's Gam and h_prev (fp32, P x N each), dt and its share of the group's B and C rows;
    write dx (fp32), the per-head dB and dC (fp32, Q x N each), ddt and the chunk's dA and dD
    partials."""
    e = 2 if wl.dtype == "bf16" else 4
    reads = 2 * Q * wl.P * e + 2 * wl.P * wl.N * 4 + Q * 4 + 2 * Q * wl.N * e * wl.G / wl.H
    writes = Q * wl.P * 4 + 2 * Q * wl.N * 4 + Q * 4 + 8
    return reads + writes


def bwd_grad_mma_flops_per_chunk_head(P, N, Q=64):
    """Issued dense bf16 MMA flops of one (chunk, head) in the tensor-core gradient kernel:
    C B^T and dy x^T; B Gam^T, C h_prev^T, Gam^T x^T and h_prev^T dy^T over the three bf16
    pieces of Gam and h_prev; the three intra-chunk products over the two pieces of the
    masked operand."""
    return 2 * Q * Q * N + 2 * Q * Q * P + 3 * 4 * (2 * Q * P * N) + 2 * (2 * Q * Q * P + 2 * 2 * N * Q * Q)


def bwd_grad_roofline(wl, ms_per_launch):
    """Roofline of the gradient kernel: on the tensor-core form (bf16, P = 64, N = 128) the
    bytes it must move against the HBM peak, with its issued MMA flops beside them; on the
    CUDA-core form its fp32 multiply-add flops against the CUDA cores' FMA issue."""
    units = -(-wl.L // 64) * wl.H * wl.b
    if wl.dtype == "bf16" and wl.P == 64 and wl.N == 128:
        peak, peak_src = hbm_peak()
        tpeak, tpeak_src = bf16_peak()
        alg = bwd_grad_bytes_per_chunk_head(wl) * units
        achieved = alg / (ms_per_launch / 1e3) / 1e9
        tflops = bwd_grad_mma_flops_per_chunk_head(wl.P, wl.N) * units / (ms_per_launch / 1e3) / 1e12
        traffic_pt = recorded_traffic("bwd_chunk_grad_tc")
        return {"bound": "hbm", "kernel": "bwd_chunk_grad_tc", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "peak_source": peak_src,
                "traffic": None if traffic_pt is None else traffic_pt * wl.L * wl.b,
                "algorithmic_bytes_per_launch": alg, "tensor_achieved_tflops": tflops,
                "tensor_peak_tflops": tpeak, "tensor_frac": tflops / tpeak, "tensor_peak_source": tpeak_src,
                "tensor_flops": "issued dense bf16 MMA flops of the kernel"}
    _, f_grad = bwd_flops_per_chunk_head(wl.P, wl.N)
    grad_flops = f_grad * units
    achieved = grad_flops / (ms_per_launch / 1e3) / 1e12
    return {"bound": "alu", "kernel": "bwd_chunk_grad", "achieved": achieved, "peak": FP32_ALU_TFLOPS,
            "unit": "TFLOP/s", "frac": achieved / FP32_ALU_TFLOPS,
            "peak_source": "derived: 148 SMs x 128 fp32 FMA lanes x 2 x 1.965 GHz", "traffic": None,
            "algorithmic_flops_per_launch": grad_flops}


def run_backward(args, world, rank, local):
    """Gradients through the scan from the forward's checkpoints (cell recompute), timed
    with CUDA events like the headline step; the forward runs once, before the timing."""
    import __graft_entry__
    __graft_entry__.build()
    import mamba_selective_state_causal_b200 as ssd
    wl = ssd_synth.BY_NAME["mamba2-0.3b-L16k"]
    d = torch.device("cuda", torch.cuda.current_device())
    seed = rank_seed(wl, rank)
    prm = ssd_synth.make_params(wl, device=d, seed=seed)
    dt = ssd_synth.make_dt(wl, prm["dt_bias"], device=d, seed=seed)
    x, Bm, Cm = ssd_synth.make_xbc(wl, device=d, seed=seed)
    dy, dhf = ssd_synth.make_grads(wl, device=d, seed=seed)
    _, _, ck = ssd.scan_forward(x, Bm, Cm, dt, prm["A"], prm["D"], H=wl.H, Q=wl.Q, s=wl.s)
    ws = torch.empty(ssd.backward_workspace_size(wl.b, wl.L, wl.H, wl.P, wl.N), dtype=torch.uint8, device=d)
    out = {"dx": torch.empty(wl.b, wl.L, wl.H, wl.P, device=d), "dB": torch.empty(wl.b, wl.L, wl.G, wl.N, device=d),
           "dC": torch.empty(wl.b, wl.L, wl.G, wl.N, device=d), "ddt": torch.empty(wl.b, wl.L, wl.H, device=d),
           "dA": torch.empty(wl.H, device=d), "dD": torch.empty(wl.H, device=d),
           "dh0": torch.empty(wl.b, wl.H, wl.P, wl.N, device=d)}

    def step():
        ssd.scan_backward(x, Bm, Cm, dt, prm["A"], prm["D"], dy, h_ckpt=ck, dh_final=dhf, H=wl.H, G=wl.G,
                          s=wl.s, workspace=ws, out=out)

    clocks = clock_sampler(local)
    clocks.start()
    ms = time_steps(step, args.steps, args.warmup, world, local)
    clk = clocks.stop()
    ssd.sync_status()
    ms = max_over_ranks(world, ms)
    ssd.profile_begin()
    prof_steps = min(args.steps, 5)
    for _ in range(prof_steps):
        step()
    torch.cuda.synchronize()
    prof = ssd.profile_end()
    per_launch = {k: v["total_ms"] / v["launches"] for k, v in prof.items()}
    nch = -(-wl.L // 64)
    f_sum, f_grad = bwd_flops_per_chunk_head(wl.P, wl.N)
    step_flops = (f_sum + f_grad) * nch * wl.H * wl.b
    line = {
        "metric": "SSD scan backward tokens/s (0.3B shape, L=16384, cells recomputed from checkpoints)",
        "value": wl.tokens * world * args.steps / (ms / 1e3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": wl.name + "-backward", "batch": wl.b, "seq_len": wl.L, "heads": wl.H,
                   "headdim": wl.P, "d_state": wl.N, "ckpt_stride": wl.s, "io_dtype": wl.dtype,
                   "l2": "workspace and outputs larger than L2 (%.1f GB)" % (ws.numel() / 1e9)},
        "roofline": bwd_grad_roofline(wl, per_launch["bwd_chunk_grad"]),
        "step_flops": step_flops,
        "kernels": {k: {"launches_per_step": v["launches"] / prof_steps, "ms_per_launch": per_launch[k]}
                    for k, v in prof.items()},
        # per step: summary, two chains, gradients, two reductions
        "gpu_launches": 6 * args.steps,
        "clocks": clk,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_layer_backward(args, world, rank, local):
    """Gradients through the whole layer (conv1d + SiLU, then the scan) from the forward's state
    checkpoints and conv buffers (each cell of s tokens rebuilt on its own), timed with CUDA
    events like the headline step; the forward runs once, before the timing."""
    import __graft_entry__
    __graft_entry__.build()
    import mamba_selective_state_causal_b200 as ssd
    wl = ssd_synth.BY_NAME["mamba2-0.3b-L16k"]
    d = torch.device("cuda", torch.cuda.current_device())
    seed = rank_seed(wl, rank)
    prm = ssd_synth.make_params(wl, device=d, seed=seed)
    u = ssd_synth.make_u(wl, device=d, seed=seed)
    dt = ssd_synth.make_dt(wl, prm["dt_bias"], device=d, seed=seed)
    dy, dhf = ssd_synth.make_grads(wl, device=d, seed=seed)
    dto, _ = ssd_synth.make_conv_grads(wl, device=d, seed=seed)
    cc = torch.empty(wl.b, wl.L // wl.s, 3, wl.cch, dtype=u.dtype, device=d)
    fwd = ssd.stream_forward(u, prm["w"], dt, prm["A"], prm["D"], H=wl.H, P=wl.P, N=wl.N, G=wl.G, Q=wl.Q,
                             s=wl.s, conv_bias=prm["bias"], conv_ckpt=cc, keep_v=False)
    ws = torch.empty(ssd.layer_backward_workspace_size(wl.b, wl.L, wl.H, wl.P, wl.N, wl.G, ssd.SSD_BF16),
                     dtype=torch.uint8, device=d)
    kw = dict(H=wl.H, P=wl.P, N=wl.N, G=wl.G, s=wl.s, conv_bias=prm["bias"], h_ckpt=fwd["h_ckpt"],
              conv_ckpt=cc, dh_final=dhf, dtail_out=dto, workspace=ws)
    out = ssd.layer_backward(u, prm["w"], dt, prm["A"], prm["D"], dy, **kw)

    def step():
        ssd.layer_backward(u, prm["w"], dt, prm["A"], prm["D"], dy, out=out, **kw)

    clocks = clock_sampler(local)
    clocks.start()
    ms = time_steps(step, args.steps, args.warmup, world, local)
    clk = clocks.stop()
    ssd.sync_status()
    ms = max_over_ranks(world, ms)
    ssd.profile_begin()
    prof_steps = min(args.steps, 5)
    for _ in range(prof_steps):
        step()
    torch.cuda.synchronize()
    prof = ssd.profile_end()
    per_launch = {k: v["total_ms"] / v["launches"] for k, v in prof.items()}
    line = {
        "metric": "SSD layer backward tokens/s (0.3B shape, L=16384, cells rebuilt from state checkpoints "
                  "and conv buffers)",
        "value": wl.tokens * world * args.steps / (ms / 1e3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": wl.name + "-layer-backward", "batch": wl.b, "seq_len": wl.L, "heads": wl.H,
                   "headdim": wl.P, "d_state": wl.N, "ckpt_stride": wl.s, "io_dtype": wl.dtype,
                   "l2": "workspace and outputs larger than L2 (%.1f GB)" % (ws.numel() / 1e9)},
        "roofline": bwd_grad_roofline(wl, per_launch["bwd_chunk_grad"]),
        "kernels": {k: {"launches_per_step": v["launches"] / prof_steps, "ms_per_launch": per_launch[k]}
                    for k, v in prof.items()},
        # per step: the cells' conv, the scan backward's six, the conv backward and its reduction
        "gpu_launches": 9 * args.steps,
        "clocks": clk,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_gated_norm(args, world, rank, local):
    """out = rmsnorm(y * silu(z)) * w on 131072 rows of the 0.3B d_inner (2048), bf16, one group."""
    import __graft_entry__
    __graft_entry__.build()
    import mamba_selective_state_causal_b200 as ssd
    rows, d = 131072, 2048
    dev = torch.device("cuda", torch.cuda.current_device())
    g = torch.Generator(device=dev)
    g.manual_seed(100 * rank + 7)
    y = torch.randn(rows, d, device=dev, generator=g).to(torch.bfloat16)
    z = torch.randn(rows, d, device=dev, generator=g).to(torch.bfloat16)
    w = torch.randn(d, device=dev, generator=g)
    out = torch.empty_like(y)

    def step():
        ssd.gated_rmsnorm(y, z, w, eps=1e-5, out=out)

    clocks = clock_sampler(local)
    clocks.start()
    ms = time_steps(step, args.steps, args.warmup, world, local)
    clk = clocks.stop()
    ssd.sync_status()
    ms = max_over_ranks(world, ms)
    step_bytes = rows * d * 2 * 3
    peak, peak_src = hbm_peak()
    achieved = step_bytes / (ms / args.steps / 1e3) / 1e9
    line = {
        "metric": "gated RMS norm rows/s (0.3B d_inner = 2048, bf16)",
        "value": rows * world * args.steps / (ms / 1e3), "unit": "rows/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "gated-rmsnorm-0.3b-131072rows", "rows": rows, "d": d, "group": d,
                   "l2": "inputs larger than L2 (%.2f GB)" % (2 * rows * d * 2 / 1e9)},
        "roofline": {"bound": "hbm", "kernel": "gated_rmsnorm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_source": peak_src, "traffic": None,
                     "algorithmic_bytes_per_launch": step_bytes},
        "gpu_launches": args.steps,
        "clocks": clk,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    wl = ssd_synth.BY_NAME[args.workload]
    if args.seq_len or args.segments:
        wl = ssd_synth.scaled(wl, L=args.seq_len or wl.L, segments=args.segments or wl.segments,
                              name=wl.name + f"-profile-L{args.seq_len or wl.L}")
    world, rank, local = dist_setup()
    if args.impl == "reference":
        run_reference(args, wl, world, rank)
        return
    if args.decode_streams > 0:
        run_decode(args, world, rank, local)
        return
    if args.backward:
        run_backward(args, world, rank, local)
        return
    if args.layer_backward:
        run_layer_backward(args, world, rank, local)
        return
    if args.gated_norm:
        run_gated_norm(args, world, rank, local)
        return
    import __graft_entry__
    __graft_entry__.build()
    layer = Layer(wl, seed=rank_seed(wl, rank), fused=not args.two_call)

    clocks = clock_sampler(local)
    clocks.start()
    ms = time_steps(layer.step, args.steps, args.warmup, world, local)
    clk = clocks.stop()
    layer.ssd.sync_status()
    ms = max_over_ranks(world, ms)
    ms_step = ms / args.steps
    value = job_throughput(wl, world, args.steps, ms)

    # per-kernel times over a second, profiled pass of the same steps
    layer.ssd.profile_begin()
    prof_steps = min(args.steps, 5)
    for _ in range(prof_steps):
        layer.step()
    torch.cuda.synchronize()
    prof = layer.ssd.profile_end()
    launches_per_step = sum(v["launches"] for v in prof.values()) / prof_steps

    conv_b, scan_b = algorithmic_bytes_per_token(wl)
    e = 2 if wl.dtype == "bf16" else 4
    fused = layer.fused and "stripe_state_tc" in prof
    peak, peak_src = hbm_peak()
    tpeak, tpeak_src = bf16_peak()
    per_launch = {k: v["total_ms"] / v["launches"] for k, v in prof.items()}
    dom = max(prof, key=lambda k: prof[k]["total_ms"])
    tokens_per_launch = {
        "conv1d_silu": wl.b * wl.seg_len, "chunk_output_tc": wl.b * wl.seg_len,
        "chunk_output_generic": wl.b * wl.seg_len, "stripe_state_tc": wl.b * wl.seg_len,
        "stripe_state_generic": wl.b * wl.seg_len}
    alg_per_token = {
        # the conv kernel reads u and writes v: all channels, or only B/C's on the fused path
        "conv1d_silu": 2 * 2 * wl.G * wl.N * e if fused else conv_b,
        # the output pass reads x (or u's x columns), B, C, dt and writes y and the checkpoints
        "chunk_output_tc": scan_b, "chunk_output_generic": scan_b,
        # pass A's own necessary reads: x (u's x columns on the fused path, where it also
        # writes the conv output of x), B, dt
        "stripe_state_tc": (2 if fused else 1) * wl.d_inner * e + wl.G * wl.N * e + 4 * wl.H,
        "stripe_state_generic": wl.d_inner * e + wl.G * wl.N * e + 4 * wl.H}
    dom_alg = alg_per_token.get(dom, 0) * tokens_per_launch.get(dom, 0)
    achieved = dom_alg / (per_launch[dom] / 1e3) / 1e9
    traffic_pt = recorded_traffic(dom)
    roofline = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "peak_source": peak_src,
                "traffic": None if traffic_pt is None else traffic_pt * tokens_per_launch.get(dom, 0),
                "algorithmic_bytes_per_launch": dom_alg}
    if dom == "chunk_output_tc":
        tflops = issued_mma_flops_per_token(wl) * tokens_per_launch[dom] / (per_launch[dom] / 1e3) / 1e12
        roofline.update({"tensor_achieved_tflops": tflops, "tensor_peak_tflops": tpeak,
                         "tensor_frac": tflops / tpeak, "tensor_peak_source": tpeak_src,
                         "tensor_flops": "issued dense bf16 MMA flops of the kernel"})
    # the whole step: the bytes the layer must move (read u and dt, write y and checkpoints)
    # and, for the target as stated, the two-call path's bytes (conv output written and re-read)
    layer_b = layer_bytes_per_token(wl)
    step_bytes = layer_b * wl.tokens
    step_frac = step_bytes / (ms_step / 1e3) / 1e9 / peak
    two_call_frac = (conv_b + scan_b) * wl.tokens / (ms_step / 1e3) / 1e9 / peak
    kernels = {k: {"launches_per_step": v["launches"] / prof_steps, "ms_per_launch": per_launch[k],
                   "share": v["total_ms"] / sum(x["total_ms"] for x in prof.values())}
               for k, v in prof.items()}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, args.cpu_sample_tokens)
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(layer)
        if world > 1:
            e2e_ms = max_over_ranks(world, e2e["ms_per_step"])
            e2e["value"] = wl.tokens * world / (e2e_ms / 1e3)

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": wl.name, "batch": wl.b, "seq_len": wl.L, "segments": wl.segments,
                   "heads": wl.H, "headdim": wl.P, "d_state": wl.N, "chunk": wl.Q,
                   "ckpt_stride": wl.s, "parallelism": f"replicas{world}",
                   "l2": layer.l2_note},
        "roofline": roofline,
        "step_roofline": {"bound": "hbm", "algorithmic_bytes_per_token": layer_b,
                          "achieved": step_bytes / (ms_step / 1e3) / 1e9, "peak": peak, "frac": step_frac,
                          "two_call_bytes_per_token": conv_b + scan_b, "two_call_frac": two_call_frac,
                          "path": "fused conv" if fused else "two-call"},
        "kernels": kernels,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": int(round(launches_per_step * args.steps)),
        "clocks": clk,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
