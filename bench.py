"""Benchmark of the fused attention hot path (forward + backward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one forward and one backward pass (every stage of the hot path)
over one batch of the causal decoder workload: BNSD bf16, B=4, N=32,
S=2048, D=128, scale 1/sqrt(128), causal mask, dO ~ N(0, 1).  Inputs are
synthetic, seeded, and resident in HBM; together they exceed the 126 MB L2,
so no flush is needed between steps.

FLOPs follow the usual convention: 4*B*N*Sq*Sk*D for the forward, 2.5x that
for the backward, halved under the causal mask.  The metric is whole-job
TFLOP/s (fwd+bwd), with the forward-only rate and both fractions of the
measured dense bf16 tensor peak reported alongside.

--impl reference times the fp64 CPU oracle (the reference implementation of
the method) on a bounded sample of the same workload on this host's cores.

Multi-GPU (torchrun): every rank runs the same workload on its own GPU (the
operator shards over (b, h) with no data exchange: replicas, weak scaling);
timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

B, N, S, D = 4, 32, 2048, 128
WORKLOAD = "causal self-attention fwd+bwd, BNSD bf16, B=4 N=32 S=2048 D=128"
METRIC = "fused attention TFLOP/s (fwd, fwd+bwd) and % of B200 dense BF16 peak"
FWD_FLOPS = 4.0 * B * N * S * S * D / 2.0
BWD_FLOPS = 2.5 * FWD_FLOPS
STEP_FLOPS = FWD_FLOPS + BWD_FLOPS
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0,
                  "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = ["attention_fwd_bwd_02_b200/csrc/fwd_sm100.cu",
                  "attention_fwd_bwd_02_b200/csrc/bwd_sm100.cu",
                  "attention_fwd_bwd_02_b200/csrc/aux.cu",
                  "attention_fwd_bwd_02_b200/csrc/ptx.cuh",
                  "attention_fwd_bwd_02_b200/csrc/sched.cuh",
                  "attention_fwd_bwd_02_b200/csrc/philox.cuh",
                  "attention_fwd_bwd_02_b200/csrc/fa_common.cuh"]


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def source_hash():
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def committed_ncu():
    """Per-launch figures from the committed ncu summary, if it was taken on
    the current kernel sources (else empty): DRAM bytes per kernel call
    ("kernels") and per kernel duration, DRAM GB/s and tensor-pipe activity
    ("ncu")."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return {}, {}
    if d.get("source_hash") != source_hash():
        return {}, {}
    return d.get("kernels", {}), d.get("ncu", {})


_SAMPLER = r"""
import sys, time
import pynvml as nv
nv.nvmlInit()
bus = sys.argv[1]
try:
    h = nv.nvmlDeviceGetHandleByPciBusId(bus)
except Exception:
    h = nv.nvmlDeviceGetHandleByIndex(int(sys.argv[2]))
mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
period = float(sys.argv[3])
out = sys.stdout
while True:
    try:
        pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
    except Exception:
        pw = -1.0
    out.write("%d %d %.1f %d\n" % (nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM), mx, pw,
                                    nv.nvmlDeviceGetCurrentClocksEventReasons(h)))
    out.flush()
    time.sleep(period)
"""


class ClockSampler:
    """Samples SM clocks, power and clock-event (throttle) reasons through
    NVML every 2 ms while the GPU works.  The sampler is a separate process,
    so the benchmark's own Python thread cannot starve it."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, cuda_index, period_s=0.002):
        self.cuda_index = cuda_index
        self.period = period_s
        self.samples = []          # (sm_mhz, max_mhz, power_w, reason_bits)
        self.error = None
        self.proc = None
        self._reader = None
        self._on = False

    def _bus_id(self):
        import torch
        p = torch.cuda.get_device_properties(self.cuda_index)
        return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"

    def _read(self):
        for line in self.proc.stdout:
            parts = line.split()
            if len(parts) == 4 and self._on:
                try:
                    pw = float(parts[2])
                    self.samples.append((int(parts[0]), int(parts[1]),
                                         pw if pw >= 0 else None, int(parts[3])))
                except ValueError:
                    pass

    def start(self):
        """Launch the sampler (its first samples arrive after it imports NVML)."""
        import subprocess
        try:
            self.proc = subprocess.Popen(
                [sys.executable, "-c", _SAMPLER, self._bus_id(), str(self.cuda_index),
                 str(self.period)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError as e:
            self.error = f"sampler did not start: {e}"
            return self
        self._reader = threading.Thread(target=self._read, daemon=True)
        self._reader.start()
        return self

    def record(self, on):
        """Keep samples only while `on` (the warm-up and the timed region)."""
        self._on = on

    def stop(self):
        self._on = False
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self._reader is not None:
            self._reader.join(timeout=5)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "source": "nvml", "error": self.error or "no samples"}
        try:
            import pynvml as nv
            consts = [(n, getattr(nv, c, 0)) for n, c in self.REASONS]
        except ImportError:
            consts = []
        reasons = set()
        for *_, bits in self.samples:
            for name, c in consts:
                if bits & c:
                    reasons.add(name)
        power = [s[2] for s in self.samples if s[2] is not None]
        return {"sm_mhz": statistics.median(s[0] for s in self.samples),
                "sm_min_mhz": min(s[0] for s in self.samples),
                "sm_max_mhz": max(s[1] for s in self.samples),
                "power_w_median": round(statistics.median(power), 1) if power else None,
                "reasons": sorted(reasons), "samples": len(self.samples),
                "source": "nvml in a separate process, 2 ms period, warm-up and timed region"}


def dist_setup(n_gpus, backend=None):
    """Joins the process group of a torchrun launch (one rank per GPU).  The
    backend is NCCL on GPUs; gloo serves the CPU tests of this plumbing."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        import torch
        backend = backend or "nccl"
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=timedelta(seconds=120))
    return rank, world, local


def _collective_device():
    import torch
    import torch.distributed as dist
    return torch.device("cuda", torch.cuda.current_device()) \
        if dist.get_backend() == "nccl" else torch.device("cpu")


def max_over_ranks(x, world):
    """The largest of every rank's x (each rank's own device timing)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=_collective_device())
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def whole_job_value(step_flops_per_rank, world, ms_per_step):
    """Whole-job throughput (TFLOP/s): every rank runs the same workload
    (weak scaling), the step time is the slowest rank's."""
    return step_flops_per_rank * world / (ms_per_step * 1e-3) / 1e12


def run_ours(args):
    import torch
    from attention_fwd_bwd_02_b200 import fa
    from attention_fwd_bwd_02_b200 import inputs as I

    rank, world, local = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    case = I.config2()
    q, k, v, do = (t.to(dev) for t in (case.q, case.k, case.v, case.dout))
    scale = case.scale
    shape = fa.make_shape(q, k, N, "BNSD")
    ws = torch.empty(fa.bwd_workspace_size(shape), dtype=torch.uint8, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty(B, N, S, dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    stream = torch.cuda.current_stream(dev)

    def fwd():
        fa.fwd(q, k, v, N, "BNSD", scale=scale, causal=True, out=out, lse=lse)

    def bwd():
        fa.bwd(q, k, v, out, do, lse, N, "BNSD", scale=scale, causal=True,
               workspace=ws, dq=dq, dk=dk, dv=dv)

    # Clocks are sampled from the warm-up on, so that even a short timed
    # region sees several samples of the loaded GPU.
    clk = ClockSampler(local).start()
    time.sleep(1.0)  # the sampler imports NVML before its first sample
    clk.record(True)
    for _ in range(args.warmup):
        fwd()
        bwd()
    fa.sync_status(dev)

    # --- device-resident timing: per-step events around fwd and bwd
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    if True:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for s in range(args.steps):
            ev[s][0].record(stream)
            fwd()
            ev[s][1].record(stream)
            bwd()
            ev[s][2].record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
    clk.stop()
    fa.sync_status(dev)
    total_ms = t0.elapsed_time(t1)
    fwd_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / args.steps
    bwd_ms = sum(e[1].elapsed_time(e[2]) for e in ev) / args.steps
    total_ms = max_over_ranks(total_ms, world)
    fwd_ms = max_over_ranks(fwd_ms, world)
    bwd_ms = max_over_ranks(bwd_ms, world)
    barrier(world)

    # --- end to end through the public API with host buffers.  Every step
    # copies its inputs from pinned host memory and reads its results back.
    # Two device buffer sets and three streams pipeline the steps: the
    # inputs of step n+1 go up and the results of step n-1 come down (PCIe
    # is full duplex) while step n computes.
    pin = {n: t.pin_memory() for n, t in (("q", case.q), ("k", case.k), ("v", case.v),
                                          ("do", case.dout))}
    host_out = {n: torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
                for n, t in (("out", out), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv))}
    h2d = sum(t.numel() * t.element_size() for t in pin.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())
    sets = [dict(q=q, k=k, v=v, do=do, out=out, lse=lse, dq=dq, dk=dk, dv=dv)]
    sets.append({n: torch.empty_like(t) for n, t in sets[0].items()})
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    s_cmp = stream
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for e in ev_cmp + ev_out:
        e.record(s_cmp)

    def e2e_step(t):
        b = sets[t % 2]
        s_in.wait_event(ev_cmp[t % 2])          # step t-2 has read these inputs
        with torch.cuda.stream(s_in):
            for n in ("q", "k", "v", "do"):
                b[n].copy_(pin[n], non_blocking=True)
            ev_in[t % 2].record(s_in)
        s_cmp.wait_event(ev_in[t % 2])
        s_cmp.wait_event(ev_out[t % 2])         # step t-2's results are down
        with torch.cuda.stream(s_cmp):
            fa.fwd(b["q"], b["k"], b["v"], N, "BNSD", scale=scale, causal=True,
                   out=b["out"], lse=b["lse"])
            fa.bwd(b["q"], b["k"], b["v"], b["out"], b["do"], b["lse"], N, "BNSD",
                   scale=scale, causal=True, workspace=ws, dq=b["dq"], dk=b["dk"], dv=b["dv"])
            ev_cmp[t % 2].record(s_cmp)
        s_out.wait_event(ev_cmp[t % 2])
        with torch.cuda.stream(s_out):
            for n in ("out", "lse", "dq", "dk", "dv"):
                host_out[n].copy_(b[n], non_blocking=True)
            ev_out[t % 2].record(s_out)

    for t in range(max(2, args.warmup)):
        e2e_step(t)
    barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for t in range(args.steps):
        e2e_step(t)
    e1.record(s_out)
    torch.cuda.synchronize()
    fa.sync_status(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world) / args.steps

    if rank != 0:
        finish(world)
        return
    pk, pk_kind = peaks()
    ms_step = total_ms / args.steps
    value = whole_job_value(STEP_FLOPS, world, ms_step)
    fwd_tf = FWD_FLOPS / (fwd_ms * 1e-3) / 1e12
    bwd_tf = BWD_FLOPS / (bwd_ms * 1e-3) / 1e12
    peak_burst = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    peak_sust = pk.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    traffic, ncu = committed_ncu()
    dominant = "bwd" if bwd_ms >= fwd_ms else "fwd"

    def roof(kind, tf, ms):
        return {"kernel": "fa_fwd (fwd_sm100)" if kind == "fwd" else
                "fa_bwd (bwd_pre + bwd_sm100 + bwd_post)",
                "bound": "tensor", "achieved": round(tf, 1), "peak": peak_burst,
                "unit": "TFLOP/s", "frac": round(tf / peak_burst, 4),
                "peak_kind": f"{pk_kind} bf16_tflops (burst)",
                "frac_of_sustained": round(tf / peak_sust, 4),
                "frac_of_nominal_2250": round(tf / 2250.0, 4),
                "ms_per_launch": round(ms, 4),
                "algorithmic_flops": FWD_FLOPS if kind == "fwd" else BWD_FLOPS,
                "traffic": traffic.get(kind),
                "ncu": ({"fwd_sm100": ncu.get("fwd")} if kind == "fwd" else
                        {"bwd_pre": ncu.get("bwd_pre"), "bwd_sm100": ncu.get("bwd_main"),
                         "bwd_post": ncu.get("bwd_post")}) if ncu else None}

    cpu = cpu_baseline(args) if not args.no_cpu_baseline else None
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1), resident in HBM)",
        "config": {"workload": WORKLOAD, "B": B, "N": N, "S": S, "D": D,
                   "mask": "causal", "scale": "1/sqrt(128)",
                   "parallelism": f"replicas x{world} (no data-path collective)",
                   "l2": "inputs exceed L2 (335 MB > 126 MB), no flush"},
        "fwd_tflops": round(fwd_tf, 2),
        "bwd_tflops": round(bwd_tf, 2),
        "fwd_ms": round(fwd_ms, 4),
        "bwd_ms": round(bwd_ms, 4),
        "fwd_frac_of_peak": round(fwd_tf / peak_burst, 4),
        "fwd_frac_of_nominal_2250": round(fwd_tf / 2250.0, 4),
        "roofline": roof(dominant, bwd_tf if dominant == "bwd" else fwd_tf,
                         bwd_ms if dominant == "bwd" else fwd_ms),
        "roofline_fwd": roof("fwd", fwd_tf, fwd_ms),
        "cpu_baseline": cpu,
        "e2e": {"value": round(whole_job_value(STEP_FLOPS, world, e2e_ms), 2),
                "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms, 4),
                "pipelining": "pinned host buffers; two device buffer sets and three "
                              "streams: step n+1's inputs go up and step n-1's results "
                              "come down while step n computes"},
        "gpu_launches": 4 * args.steps,
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)
    finish(world)


def finish(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def oracle_sample(n_heads, seq):
    """fwd+bwd of the oracle on n_heads heads of the workload's operator
    (causal, D=128, scale 1/sqrt(128)) over a seq-token prefix.  Returns
    (seconds, algorithmic flops of the sample, threads used)."""
    import oracle
    from attention_fwd_bwd_02_b200 import inputs as I
    case = I.make_case("oracle_sample", 1, n_heads, seq, seq, D, seed=1002, causal=True)
    f64 = lambda t: t.double().numpy()
    q, k, v, do = f64(case.q), f64(case.k), f64(case.v), f64(case.dout)
    threads = min(len(os.sched_getaffinity(0)), n_heads)
    oracle.set_threads(threads)
    t = time.perf_counter()
    oracle.fwd(q, k, v, case.scale, causal=True)
    oracle.bwd(q, k, v, do, case.scale, causal=True)
    dt = time.perf_counter() - t
    flops = 3.5 * 4.0 * n_heads * seq * seq * D / 2.0
    return dt, flops, threads


def sample_heads(args, per_core):
    if args.cpu_heads > 0:
        return args.cpu_heads
    return per_core * len(os.sched_getaffinity(0))


def cpu_baseline(args):
    n = sample_heads(args, 24)
    dt, flops, threads = oracle_sample(n, args.cpu_seq)
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": threads,
            "kind": "oracle",
            "sample": f"{n} heads of the workload's operator (causal, D={D}) over a "
                      f"{args.cpu_seq}-token prefix, fwd+bwd in fp64, {dt:.1f} s",
            "seconds": round(dt, 2)}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    times, flops_s = [], 0.0
    n = sample_heads(args, 1)
    threads = 1
    for _ in range(min(args.warmup, 1)):
        oracle_sample(1, args.cpu_seq)
    for _ in range(args.steps):
        dt, fl, threads = oracle_sample(n, args.cpu_seq)
        times.append(dt)
        flops_s = fl
    ms = 1e3 * sum(times) / len(times)
    value = flops_s / (ms * 1e-3) / 1e12
    line = {
        "impl": "reference",
        "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (seeded N(0,1))",
        "config": {"workload": WORKLOAD, "B": B, "N": N, "S": S, "D": D,
                   "mask": "causal", "parallelism": "host cores (OpenMP over heads)"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads,
                         "kind": "oracle",
                         "sample": f"each step: {n} heads of the workload's operator "
                                   f"(causal, D={D}) over a {args.cpu_seq}-token prefix, "
                                   "fwd+bwd in fp64"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def _allowed_pairs(case):
    """Visible (query, key) pairs of a case, summed over (b, h), from its
    integer side inputs (padding lengths, modality ids, causal rule)."""
    import torch
    B, N, Sq, Sk = case.B, case.N, case.Sq, case.Sk
    total = 0
    for b in range(B):
        nk = Sk if case.kv_len is None else max(0, min(Sk, int(case.kv_len[b])))
        vis = torch.zeros(Sq, Sk, dtype=torch.bool)
        vis[:, :nk] = True
        if case.causal:
            vis &= torch.ones(Sq, Sk, dtype=torch.bool).tril()
        if case.modality_ids is not None:
            ids = case.modality_ids[b].long() & 1
            allow = torch.tensor(case.allow, dtype=torch.bool)
            rule = allow[ids[:, None], ids[None, :]]
            if case.allow_diag:
                rule |= torch.eye(Sq, Sk, dtype=torch.bool)
            vis &= rule
        total += int(vis.sum()) * N
    return total


def run_configs(args):
    """Times fa_fwd and fa_fwd + fa_bwd on every workload of the source pages
    (one JSON line each, after the main line's format): nominal and
    allowed-pair TFLOP/s, GB/s on the algorithmic bytes, and the fraction of
    the measured peak.  HBM-bound workloads are timed with L2 flushed
    between repetitions (a 256 MB write)."""
    import statistics as st
    import torch
    from attention_fwd_bwd_02_b200 import fa
    from attention_fwd_bwd_02_b200 import inputs as I
    pk, pk_kind = peaks()
    peak = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    cases = [("1", I.config1(), False), ("2", I.config2(), False),
             ("3a", I.config3(24), True), ("3b", I.config3(320), True),
             ("4a", I.config4(256), True), ("4b", I.config4(512), True)]
    cases += [(f"5 S={s} D={d}", I.config5(s, d), s <= 1024) for s, d in I.CONFIG5_SWEEP]
    for label, c, do_flush in cases:
        dev = {n: (None if getattr(c, n) is None else getattr(c, n).cuda())
               for n in ("q", "k", "v", "dout")}
        kw = dict(pse=None if c.slopes is None else c.slopes.cuda(), scale=c.scale,
                  causal=c.causal,
                  padding_kv_len=None if c.kv_len is None else c.kv_len.cuda())
        if c.modality_ids is not None:
            kw.update(modality_ids=c.modality_ids.cuda(), allow=c.allow, allow_diag=c.allow_diag)
        q, k, v, do = dev["q"], dev["k"], dev["v"], dev["dout"]
        out, lse = fa.fwd(q, k, v, c.N, c.layout, **kw)
        ws = torch.empty(fa.bwd_workspace_size(fa.make_shape(q, k, c.N, c.layout)),
                         dtype=torch.uint8, device="cuda")
        fwd = lambda: fa.fwd(q, k, v, c.N, c.layout, out=out, lse=lse, **kw)
        bwd = lambda: fa.bwd(q, k, v, out, do, lse, c.N, c.layout, workspace=ws, **kw)

        def timed(fn, reps=30, warm=10):
            """(device ms, call ms): the device time of one call, with the
            call queued behind a GPU spin so that the host's marshalling
            and launch cost stay off the events; and the time per call of
            back-to-back calls, which includes that host cost when it
            exceeds the device time."""
            for _ in range(warm):
                fn()
            ts = []
            for _ in range(reps):
                if do_flush:
                    flush.fill_(1)
                torch.cuda._sleep(1_000_000)  # about 0.5 ms of GPU spin
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record()
                fn()
                e1.record()
                torch.cuda.synchronize()
                ts.append(e0.elapsed_time(e1))
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            for _ in range(reps):
                fn()
            torch.cuda.synchronize()
            return st.median(ts), (time.perf_counter() - t0) * 1e3 / reps

        f_ms, f_call = timed(fwd)
        b_ms, b_call = timed(bwd)
        fa.sync_status()
        nominal = 4.0 * c.B * c.N * c.Sq * c.Sk * c.D / (2.0 if c.causal else 1.0)
        allowed = 4.0 * c.D * _allowed_pairs(c)
        esz = q.element_size()
        rows_q, rows_k = c.B * c.N * c.Sq, c.B * c.N * c.Sk
        fwd_bytes = (2 * rows_q + 2 * rows_k) * c.D * esz + 4 * rows_q
        bwd_bytes = (4 * rows_q + 4 * rows_k) * c.D * esz + 4 * rows_q
        line = {"metric": METRIC, "config": c.name, "label": label,
                "dtype": {torch.bfloat16: "bf16", torch.float32: "f32"}[q.dtype],
                "fwd_ms": round(f_ms, 4), "bwd_ms": round(b_ms, 4),
                "fwd_call_ms": round(f_call, 4), "bwd_call_ms": round(b_call, 4),
                "fwd_tflops": round(nominal / (f_ms * 1e-3) / 1e12, 2),
                "fwd_tflops_allowed_pairs": round(allowed / (f_ms * 1e-3) / 1e12, 2),
                "bwd_tflops": round(2.5 * nominal / (b_ms * 1e-3) / 1e12, 2),
                "bwd_tflops_allowed_pairs": round(2.5 * allowed / (b_ms * 1e-3) / 1e12, 2),
                "fwd_frac_of_peak": round(nominal / (f_ms * 1e-3) / 1e12 / peak, 4),
                "fwd_gbs": round(fwd_bytes / (f_ms * 1e-3) / 1e9, 1),
                "bwd_gbs": round(bwd_bytes / (b_ms * 1e-3) / 1e9, 1),
                "peak": peak, "peak_kind": f"{pk_kind} bf16_tflops (burst)",
                "l2_flushed_between_reps": do_flush,
                "timing": "fwd_ms/bwd_ms: device time, median of 30 after 10 warm-ups, each call "
                          "queued behind a GPU spin; *_call_ms: back-to-back calls incl. host cost "
                          "(no L2 flush)"}
        print(json.dumps(line), flush=True)
        del dev, out, lse, ws


def run_variant(args):
    """Times one NEXT-row variant of the headline workload (causal B=4 N=32
    S=2048 D=128) and prints one JSON line (not the main line):
      e4m3    -- the fp8 forward (fa_fwd with e4m3 q, k, v; bf16 out);
      dense   -- fa_fwd + fa_bwd with a dense [1, N, S, S] fp32 term;
      dropout -- fa_fwd + fa_bwd with keep_prob = 0.9;
      mask    -- fa_fwd + fa_bwd with a random [B, 1, S, S] bool mask (half
                 the pairs) on top of the causal rule, no tile map."""
    import torch
    from attention_fwd_bwd_02_b200 import fa
    from attention_fwd_bwd_02_b200 import inputs as I
    pk, pk_kind = peaks()
    peak = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    case = I.config2()
    dev = torch.device("cuda")
    q, k, v, do = (t.to(dev) for t in (case.q, case.k, case.v, case.dout))
    kw = dict(scale=case.scale, causal=True)
    with_bwd = args.variant != "e4m3"
    if args.variant == "e4m3":
        q, k, v = (t.to(torch.float8_e4m3fn) for t in (q, k, v))
        peak = 2.0 * peak   # e4m3 dense rate is twice bf16's (4.5 vs 2.25 PFLOP/s nominal)
    elif args.variant == "dense":
        g = torch.Generator(device=dev).manual_seed(3)
        kw["pse"] = torch.randn(1, N, S, S, device=dev, generator=g)
    elif args.variant == "mask":
        g = torch.Generator(device=dev).manual_seed(4)
        kw["atten_mask"] = (torch.rand(B, 1, S, S, device=dev, generator=g) < 0.5).to(torch.uint8)
    else:
        kw.update(keep_prob=0.9, seed=1234, offset=0)
    out, lse = fa.fwd(q, k, v, N, **kw)
    ws = torch.empty(fa.bwd_workspace_size(fa.make_shape(q, k, N, "BNSD")), dtype=torch.uint8,
                     device=dev)
    step = [lambda: fa.fwd(q, k, v, N, out=out, lse=lse, **kw)]
    if with_bwd:
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        step.append(lambda: fa.bwd(q, k, v, out, do, lse, N, workspace=ws, dq=dq, dk=dk,
                                   dv=dv, **kw))
    for _ in range(args.warmup):
        for f in step:
            f()
    fa.sync_status(dev)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    torch.cuda.synchronize()
    for s_ in range(args.steps):
        ev[s_][0].record()
        step[0]()
        ev[s_][1].record()
        if with_bwd:
            step[1]()
        ev[s_][2].record()
    torch.cuda.synchronize()
    fa.sync_status(dev)
    fwd_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / args.steps
    line = {"variant": args.variant, "metric": METRIC, "unit": "TFLOP/s",
            "config": {"workload": WORKLOAD, "B": B, "N": N, "S": S, "D": D},
            "steps": args.steps, "warmup": args.warmup,
            "fwd_ms": round(fwd_ms, 4), "fwd_tflops": round(FWD_FLOPS / (fwd_ms * 1e-3) / 1e12, 2),
            "fwd_frac_of_peak": round(FWD_FLOPS / (fwd_ms * 1e-3) / 1e12 / peak, 4),
            "peak": peak, "peak_kind": f"{pk_kind} bf16_tflops (burst)"
                                       + (" x 2 for e4m3" if args.variant == "e4m3" else "")}
    if with_bwd:
        bwd_ms = sum(e[1].elapsed_time(e[2]) for e in ev) / args.steps
        line.update(bwd_ms=round(bwd_ms, 4),
                    bwd_tflops=round(BWD_FLOPS / (bwd_ms * 1e-3) / 1e12, 2))
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-heads", type=int, default=0,
                    help="(b, h) heads in the oracle's bounded sample "
                         "(default: one per host core)")
    ap.add_argument("--cpu-seq", type=int, default=512,
                    help="token prefix of the oracle's bounded sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--configs", action="store_true",
                    help="instead of the main line, time every workload of the "
                         "source pages (one JSON line each)")
    ap.add_argument("--variant", choices=["e4m3", "dense", "dropout", "mask"],
                    help="instead of the main line, time one variant of the "
                         "headline workload (fp8 forward, dense term, dropout, "
                         "bool mask)")
    args = ap.parse_args()
    if args.impl == "ours":
        args.warmup = max(3, args.warmup)   # at least 3 untimed warm-up steps
    if args.impl == "reference":
        run_reference(args)
    elif args.configs:
        run_configs(args)
    elif args.variant:
        run_variant(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
