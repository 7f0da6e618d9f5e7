#!/usr/bin/env python
"""Benchmark of the GDN recurrence on B200: tokens*heads/s and roofline fraction.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one gdn_forward call over the whole workload (default: the 720p
bidirectional workload, B=2, H=16, T=75600, dk=dv=128, bf16 inputs, fp32
state), inputs resident in HBM.  Inputs total 4.4 GB, far above the 126 MB
L2, so no flush is needed between steps.  Timing: W warm-up steps, then a
barrier + device synchronise, K steps bracketed by CUDA events on the
launching stream, synchronise + barrier, max over ranks.  With N > 1 (one
process per GPU under torchrun) every rank runs its own full workload: the
scans are independent, there is no collective on the data path (weak scaling).

Also measured, and printed on the same JSON line:
  e2e          the same metric through the library's host-buffer entry point
               (pinned host inputs; host->device copies, the kernels, and the
               device->host copy of o and the states inside the timed region),
               as a streaming loop runs it: asynchronous calls alternating
               between two streams, so call i+1's copies in overlap call i's
               kernels and copies out;
  roofline     the main kernel's algorithmic bytes / its average event-timed
               duration, against the measured HBM copy bandwidth;
  parity       rel-L2 of the last timed step's o and states against the fp64
               oracle on the first and last head, whole sequences (rank 0);
  cpu_baseline the fp64 CPU oracle on a bounded sample of the same workload
               (rank 0, N = 1 only);
  clocks       SM clock and throttle reasons sampled (NVML) during the timed
               region.
--impl reference times the CPU oracle alone (the reference arm: there is no
upstream code to run).
"""
import argparse
import hashlib
import re
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GDN tokens*heads/s (bf16, 1xB200)"
UNIT = "tokens*heads/s"


def algorithmic_bytes(wl, fp8=False):
    """Bytes a perfect kernel moves once: q, k, v, gates read and o written once
    per scan direction, plus the fp32 states (in if present, out always).  fp8
    inputs: q, k and v are one byte per element (o stays bf16)."""
    es = 2 if wl.dtype == "bf16" else 4
    es_in = 1 if fp8 else es
    ndir = 2 if wl.bidi else 1
    per_tok = ndir * ((2 * wl.dk + wl.dv) * es_in + 8) + wl.dv * es
    st = wl.dk * wl.dv * 4
    n_heads = wl.B * wl.H
    states = n_heads * st * (ndir + (1 if wl.state0 else 0))
    return wl.B * wl.H * wl.T * wl.n_chunks * per_tok + states * wl.n_chunks


def algorithmic_flops(wl, C=64):
    """Useful chunkwise MMA FLOPs (triangles counted half) per token*head*direction:
    3*C*dk + 2*C*dv + C^2/3 + 6*dk*dv."""
    ndir = 2 if wl.bidi else 1
    per = 3 * C * wl.dk + 2 * C * wl.dv + C * C / 3 + 6 * wl.dk * wl.dv
    return wl.token_heads * ndir * per


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], "measured"
    return 6650.0, 1590.0, "fallback"


# B200 nominal figures (dense bf16; HBM3e), beside the measured ones
SPEC_HBM_GBS, SPEC_BF16_TFLOPS = 8000.0, 2250.0


def workload_config(wl, world):
    """The config dict of a bench line: the workload and how it is run, the same
    for the GPU arm and the reference arm."""
    bytes_ = algorithmic_bytes(wl)
    return {"workload": wl.name, "B": wl.B, "H": wl.H, "T": wl.T, "dk": wl.dk, "dv": wl.dv,
            "mode": "bidi" if wl.bidi else ("rollout of %d causal chunks" % wl.n_chunks if wl.n_chunks > 1
                                            else "causal"),
            "n_chunks": wl.n_chunks, "token_heads_per_gpu": wl.token_heads,
            "l2": ("no flush: inputs of %.2f GB per step exceed the 126 MB L2" % (bytes_ / 1e9)
                   if bytes_ >= (1 << 30) else
                   "flushed: 512 MB written before each step (%.3f GB per step would fit in the 126 MB "
                   "L2); step time from the steps' own events" % (bytes_ / 1e9)),
            "parallelism": f"replicas x{world} (independent scans, no collective)"}


def kernel_source_sha(kernel="pool"):
    """Hash of the main kernel's device code (its source and the headers it
    includes; comments and whitespace removed), so that a recorded traffic
    figure stays tied to the kernel it was taken on.  kernel: "pool" (the pooled
    kernel, dk = dv = 128) or "single" (the single-CTA kernel)."""
    h = hashlib.sha256()
    main = "gdn_chunk_pool.cu" if kernel == "pool" else "gdn_chunk_tc.cu"
    for name in (main, "gdn_chunk_common.cuh", "sm100_ptx.cuh"):
        p = os.path.join(ROOT, "gated_delta_rule_149_b200", "csrc", name)
        if os.path.exists(p):
            src = open(p).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            src = re.sub(r"//[^\n]*", "", src)
            h.update("".join(src.split()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload, sha):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(workload)
    if not d or d.get("kernel_source_sha") != sha:
        return None
    return d.get("dram_bytes_per_launch")


class ClockSampler:
    """SM clock and clock-event (throttle) reasons during the timed region.

    An NVML thread polls every 5 ms (read-only queries) and has taken its first
    sample before the region starts, so short regions are covered too;
    nvidia-smi is the fallback where NVML cannot be loaded."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    BITS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
            "sw_power_cap": 0x4}

    def __init__(self, gpu_index, device=None):
        self.gpu = gpu_index
        self.device = device
        self.proc = None
        self.f = None
        self.thread = None
        self.samples = []
        self.max_mhz = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            import torch
            p = torch.cuda.get_device_properties(self.device if self.device is not None else self.gpu)
            bus = "%08x:%02x:%02x.0" % (p.pci_domain_id, p.pci_bus_id, p.pci_device_id)
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.gpu)

    def _start_nvml(self):
        import threading
        nv, h = self._nvml_handle()
        self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        self._stop, first = threading.Event(), threading.Event()

        def run():
            while not self._stop.is_set():
                try:
                    self.samples.append((float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)),
                                         int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))))
                except Exception:
                    break
                first.set()
                self._stop.wait(0.005)
            first.set()

        self.thread = threading.Thread(target=run, daemon=True)
        self.thread.start()
        first.wait(2.0)
        if not self.samples:
            raise RuntimeError("NVML gave no sample")

    def __enter__(self):
        try:
            self._start_nvml()
            return self
        except Exception:
            self.thread = None
            self.samples = []
        try:
            self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self._stop.set()
            self.thread.join(timeout=2.0)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if self.thread is not None:
            if not self.samples:
                return None
            reasons = sorted(n for n in self.NAMES if any(r & self.BITS[n] for _, r in self.samples))
            return {"sm_mhz": statistics.median(m for m, _ in self.samples), "sm_max_mhz": self.max_mhz,
                    "reasons": reasons, "samples": len(self.samples), "source": "nvml, 5 ms"}
        if self.f is None:
            return None
        self.f.flush()
        rows = [r.split(",") for r in open(self.f.name).read().strip().splitlines() if r.strip()]
        os.unlink(self.f.name)
        sm, mx, reasons = [], None, set()
        for r in rows:
            r = [x.strip() for x in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                continue
            for n, val in zip(self.NAMES, r[5:9]):
                if val.lower() in ("active", "1"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "source": "nvidia-smi"}


def dist_setup():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    """The maximum of a per-rank scalar over all ranks (every rank gets it)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cpu" if dist.get_backend() == "gloo" else "cuda"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(token_heads_per_rank, total_ms, steps, world):
    """Weak scaling over replicas: every rank runs its own full workload, the
    job's step time is the slowest rank's, and the job processes world times
    one rank's tokens*heads per step.  Returns (ms_per_step, value)."""
    ms_per_step = max_over_ranks(total_ms, world) / steps
    return ms_per_step, world * token_heads_per_rank / (ms_per_step * 1e-3)


# --------------------------------------------------------------------------
# CPU oracle baseline (a bounded sample of the workload)
# --------------------------------------------------------------------------

def oracle_sample_throughput(wl, inp=None, target_s=15.0):
    """Times the fp64 oracle on a bounded sample of the workload's own inputs:
    whole heads (both scan directions for bidi) truncated to a token prefix,
    sized for about target_s seconds of wall time on the host cores."""
    import oracle
    from gated_delta_rule_149_b200.inputs import make_inputs
    if inp is None:
        inp = make_inputs(wl)
    nproc = os.cpu_count() or 1
    ndir = 2 if wl.bidi else 1
    BH = wl.B * wl.H
    T_all = wl.T * wl.n_chunks
    if wl.n_chunks > 1:   # a rollout is one scan over its chunks: time it as one sequence per head
        flat = lambda t: t.movedim(0, 2).reshape(BH, T_all, *t.shape[4:])
    else:
        flat = lambda t: t.reshape(BH, *t.shape[2:])

    def run(n_heads, T):
        sl = lambda t: flat(t)[:n_heads, :T].double().numpy()[None]
        args = [sl(inp.q), sl(inp.k), sl(inp.v), sl(inp.beta), sl(inp.decay)]
        s0 = None if inp.state0 is None else inp.state0.reshape(BH, wl.dk, wl.dv)[:n_heads].double().numpy()[None]
        t0 = time.perf_counter()
        oracle.gdn_forward(*args, state_in=s0, bidi=wl.bidi, n_threads=nproc)
        return time.perf_counter() - t0

    per_wave = max(1, nproc // ndir)            # heads whose scans fill the cores once
    n_heads = min(BH, per_wave)
    T_cal = min(T_all, 2048)
    per_tok = run(n_heads, T_cal) / T_cal       # seconds per token for one wave
    T = int(min(T_all, max(256, target_s / per_tok)))
    if T == T_all:                              # whole heads are cheap: add waves
        waves = max(1, int(target_s / (per_tok * T)))
        n_heads = min(BH, per_wave * waves)
    el = run(n_heads, T)
    value = n_heads * T / el
    threads = min(nproc, n_heads * ndir)
    return {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{n_heads} of {BH} heads x first {T} of {T_all} tokens of {wl.name} "
                      f"({'both scan directions' if wl.bidi else 'causal'}), fp64, "
                      f"{el:.1f} s wall on {threads} threads",
            "elapsed_s": el, "cpu": _cpu_model()}


def sampled_parity(args, wl, inp, o_dev, s_dev, fp8=None):
    """rel-L2 of this run's GPU results (the last timed step's o and states)
    against the fp64 oracle on the same inputs, for the first and the last
    head over their whole sequences (both scan directions when bidirectional):
    the check the timing is reported beside."""
    import numpy as np
    import oracle
    if args.normalized:
        return {"checked": False,
                "why": "normalised read-out: z.q of the benchmark's signed features can be ~0; "
                       "the GPU tests check it on non-negative features"}
    BH = wl.B * wl.H
    heads = sorted({0, BH - 1})
    if wl.n_chunks > 1:   # rollout: chunk-major tensors, checked chunk by chunk
        n = wl.n_chunks
        cm = lambda t: t.reshape(n, BH, *t.shape[3:])[:, heads].double().numpy()[:, None]   # [n,1,h,..]
        t0 = time.perf_counter()
        o_ref, s_ref, _ = oracle.gdn_rollout(cm(inp.q), cm(inp.k), cm(inp.v), cm(inp.beta), cm(inp.decay),
                                             inp.state0.reshape(BH, wl.dk, wl.dv)[heads].double().numpy()[None])
        elapsed = time.perf_counter() - t0
        o = o_dev.reshape(n, BH, wl.T, wl.dv)[:, heads].double().cpu().numpy()[:, None]
        st = s_dev.reshape(BH, wl.dk, wl.dv)[heads].double().cpu().numpy()[None]
        rel = lambda x, y: float(np.linalg.norm(x - y) / np.linalg.norm(y))
        e_o = max(rel(o[c], o_ref[c]) for c in range(n))
        e_s = rel(st, s_ref)
        return {"checked": True, "rel_l2_o": e_o, "rel_l2_state": e_s, "tol": 1e-2,
                "pass": e_o <= 1e-2 and e_s <= 1e-2,
                "sample": f"heads {heads} of {BH}, all {n} chunks x {wl.T} tokens (o: worst chunk); "
                          f"fp64 oracle, {elapsed:.1f} s"}
    flat = lambda t: t.reshape(BH, *t.shape[2:])
    pick = lambda t: flat(t)[heads].double().numpy()[None]          # [1, n, ...]
    s0 = None if inp.state0 is None else pick(inp.state0)
    nproc = os.cpu_count() or 1
    t0 = time.perf_counter()
    if fp8 is not None:
        q8, k8, v8, sq, sk, sv = (t.cpu() for t in fp8)
        codes = lambda t: flat(t)[heads].numpy()[None]
        scale = lambda t: t.reshape(BH)[heads].double().numpy()[None]
        o_ref, s_ref = oracle.gdn_forward_fp8(codes(q8), codes(k8), codes(v8), scale(sq), scale(sk), scale(sv),
                                              pick(inp.beta), pick(inp.decay), state_in=s0, bidi=wl.bidi,
                                              n_threads=nproc)
    elif args.block > 0:
        o_ref, s_ref = oracle.gdn_forward_blockcausal(pick(inp.q), pick(inp.k), pick(inp.v), pick(inp.beta),
                                                      pick(inp.decay), args.block, state_in=s0, n_threads=nproc)
    else:
        o_ref, s_ref = oracle.gdn_forward(pick(inp.q), pick(inp.k), pick(inp.v), pick(inp.beta),
                                          pick(inp.decay), state_in=s0, bidi=wl.bidi, n_threads=nproc)
    elapsed = time.perf_counter() - t0
    n = len(heads)
    o = flat(o_dev)[heads].double().cpu().numpy()[None]
    if wl.bidi:
        st, st_ref = s_dev.reshape(2, BH, wl.dk, wl.dv)[:, heads], s_ref.reshape(2, n, wl.dk, wl.dv)
    else:
        st, st_ref = s_dev.reshape(BH, wl.dk, wl.dv)[heads], s_ref.reshape(n, wl.dk, wl.dv)
    st = st.double().cpu().numpy()
    rel = lambda x, y: float(np.linalg.norm(x - y) / np.linalg.norm(y))
    tol = 1e-5 if wl.dtype == "fp32" else 1e-2
    e_o, e_s = rel(o, o_ref), rel(st, st_ref)
    return {"checked": True, "rel_l2_o": e_o, "rel_l2_state": e_s, "tol": tol, "pass": e_o <= tol and e_s <= tol,
            "sample": f"heads {heads} of {BH}, all {wl.T} tokens"
                      f"{', both scan directions' if wl.bidi else ''}; fp64 oracle, {elapsed:.1f} s"}


def _cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def run_reference(args, world, rank):
    from gated_delta_rule_149_b200.inputs import WORKLOADS
    wl = WORKLOADS[args.workload]
    if rank != 0:
        return 0
    from gated_delta_rule_149_b200.inputs import make_inputs
    inp = make_inputs(wl)
    vals = []
    for i in range(args.warmup + args.steps):
        r = oracle_sample_throughput(wl, inp, target_s=args.ref_seconds)
        if i >= args.warmup:
            vals.append(r)
    value = statistics.median(v["value"] for v in vals)
    el = sum(v["elapsed_s"] for v in vals)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * el / len(vals), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(wl, world),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": vals[0]["cores"],
                             "kind": "oracle", "sample": vals[0]["sample"],
                             "cpu": vals[0]["cpu"]},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------
# GPU arm
# --------------------------------------------------------------------------

def run_gpu(args, world, rank, local):
    import torch
    from gated_delta_rule_149_b200 import (gdn, gdn_forward, gdn_forward_blockcausal, gdn_forward_fp8,
                                           gdn_forward_host_async, gdn_forward_normalized, gdn_forward_segmented,
                                           gdn_device_status, gdn_rollout)
    from gated_delta_rule_149_b200.inputs import quantize_e4m3
    from gated_delta_rule_149_b200.inputs import WORKLOADS, make_inputs

    wl = WORKLOADS[args.workload]
    rollout = wl.n_chunks > 1
    dev = torch.device("cuda", torch.cuda.current_device())
    gdn.debug_kernel_select(1 if args.kernel == "single" else 0)
    gdn.debug_plain_launch(args.plain_launch)
    inp = make_inputs(wl)
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    beta, decay = inp.beta.to(dev), inp.decay.to(dev)
    s0 = None if inp.state0 is None else inp.state0.to(dev)
    o = torch.empty(((wl.n_chunks,) if rollout else ()) + (wl.B, wl.H, wl.T, wl.dv), dtype=q.dtype, device=dev)
    s_out = torch.empty(((2,) if wl.bidi else ()) + (wl.B, wl.H, wl.dk, wl.dv),
                        dtype=torch.float32, device=dev)
    recurrent = args.recurrent or wl.dtype == "fp32"
    stream = torch.cuda.current_stream(dev)
    lib = gdn.load_library()

    # fp8 with dv = 128 runs as the one pooled kernel (codes widened in-kernel)
    fp8_prepass = args.fp8 and (wl.dv != 128 or args.kernel == "single")
    segmented = args.segments > 0 or args.block > 0 or args.normalized or fp8_prepass
    if rollout and (segmented or recurrent):
        raise SystemExit("the rollout workload runs the plain bf16 chunkwise path only")
    if args.fp8:
        if recurrent:
            raise SystemExit("--fp8 runs bf16-output workloads only")
        (q8, sq), (k8, sk), (v8, sv) = (quantize_e4m3(x) for x in (inp.q, inp.k, inp.v))
        q8, k8, v8, sq, sk, sv = (t.to(dev) for t in (q8, k8, v8, sq, sk, sv))
    if (args.segments > 0 or args.block > 0) and (wl.bidi or recurrent):
        raise SystemExit("--segments / --block run causal bf16 workloads only")
    if args.normalized and recurrent:
        raise SystemExit("--normalized runs bf16 workloads only")

    def step():
        if rollout:
            gdn_rollout(q, k, v, beta, decay, s0, o=o, state_out=s_out, stream=stream)
        elif args.fp8:
            gdn_forward_fp8(q8, k8, v8, sq, sk, sv, beta, decay, s0, bidi=wl.bidi, o=o, state_out=s_out,
                            stream=stream)
        elif args.normalized:
            gdn_forward_normalized(q, k, v, beta, decay, s0, eps=1e-6, bidi=wl.bidi, o=o, stream=stream)
        elif args.block > 0:
            gdn_forward_blockcausal(q, k, v, beta, decay, s0, block=args.block, o=o, state_out=s_out,
                                    stream=stream)
        elif args.segments > 0:
            gdn_forward_segmented(q, k, v, beta, decay, s0, n_segments=args.segments, o=o,
                                  state_out=s_out, stream=stream)
        else:
            gdn_forward(q, k, v, beta, decay, s0, bidi=wl.bidi, recurrent=recurrent, o=o,
                        state_out=s_out, stream=stream)

    for _ in range(args.warmup):
        step()
    gdn_device_status(stream)
    torch.cuda.synchronize()

    # Workloads whose bytes per step do not dwarf the 126 MB L2 are timed with
    # L2 flushed before every step (a 512 MB write, outside the step's events).
    bytes_ = algorithmic_bytes(wl, fp8=args.fp8)
    flush_buf = torch.empty(512 << 20, dtype=torch.uint8, device=dev) if bytes_ < (1 << 30) else None
    launches0 = lib.gdn_kernel_launches()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local, dev) as clk:
        t_all0 = torch.cuda.Event(enable_timing=True)
        t_all1 = torch.cuda.Event(enable_timing=True)
        t_all0.record(stream)
        for i in range(args.steps):
            if flush_buf is not None:
                flush_buf.zero_()
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        t_all1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    launches = lib.gdn_kernel_launches() - launches0
    gdn_device_status(stream)
    per_call = [a.elapsed_time(b) for a, b in ev]
    # with flushes between steps, the steps' own events give the step time
    total_ms = t_all0.elapsed_time(t_all1) if flush_buf is None else sum(per_call)
    ms_per_step, value = replica_throughput(wl.token_heads, total_ms, args.steps, world)

    # roofline of the main kernel (the plain call is one main kernel plus a tiny
    # memset; the other forms time their whole call, which "scope" says)
    hbm_peak, tc_peak, peak_kind = load_peaks()
    call_s = statistics.mean(per_call) * 1e-3
    achieved = bytes_ / call_s / 1e9
    sha = kernel_source_sha("single" if args.kernel == "single" or wl.dv != 128 or recurrent else "pool")
    traffic = recorded_traffic(wl.name, sha)
    roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved / hbm_peak, "traffic": traffic,
                "peak_kind": peak_kind, "algorithmic_bytes": bytes_,
                "frac_spec": achieved / SPEC_HBM_GBS,
                "tensor_frac_spec": algorithmic_flops(wl) / call_s / 1e12 / SPEC_BF16_TFLOPS,
                "scope": ("the token-by-token kernel (and, bidirectional, the add of its partials)"
                          if recurrent else
                          "the whole rollout call: %d chunkwise launches, one per chunk" % wl.n_chunks
                          if rollout else
                          "the chunkwise kernel (the call's one kernel)%s" % (
                              ", E4M3 codes read at one byte per element" if args.fp8 else "") if not segmented else
                          "the whole call: the bf16 kernel's algorithmic bytes over the time of all "
                          "its launches (%s)" % ("dequantising pre-pass included" if args.fp8 else
                                                 "every pass and combine included")),
                "tensor_tflops": algorithmic_flops(wl) / call_s / 1e12,
                "tensor_frac": algorithmic_flops(wl) / call_s / 1e12 / tc_peak,
                "kernel_source_sha": sha}

    # end to end through the host-buffer entry point
    pin = lambda t: t.pin_memory()
    if args.fp8:   # the host buffers of an fp8 call are its codes and scales
        hq, hk, hv, hsq, hsk, hsv = (pin(t.cpu()) for t in (q8, k8, v8, sq, sk, sv))
    else:
        hq, hk, hv = map(pin, (inp.q, inp.k, inp.v))
    hb, ha = map(pin, (inp.beta, inp.decay))
    hs0 = None if inp.state0 is None else pin(inp.state0)
    # two sets of host outputs and two streams: a streaming loop keeps one call
    # in flight while the next one's inputs upload
    e2e_streams = [stream, torch.cuda.Stream(dev)]
    hos = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for _ in range(2)]
    hsos = [torch.empty(s_out.shape, dtype=torch.float32).pin_memory() for _ in range(2)]

    def e2e_step(n):
        ho, hso = hos[n % 2], hsos[n % 2]
        if segmented or rollout or args.fp8:   # the same call on device copies of pinned host buffers
            pairs = ((hq, q8), (hk, k8), (hv, v8), (hsq, sq), (hsk, sk), (hsv, sv)) if args.fp8 else \
                ((hq, q), (hk, k), (hv, v))
            for h, dst in pairs + ((hb, beta), (ha, decay), (hs0, s0)):
                if h is not None:
                    dst.copy_(h, non_blocking=True)
            step()
            ho.copy_(o, non_blocking=True)
            hso.copy_(s_out, non_blocking=True)
        else:
            gdn_forward_host_async(hq, hk, hv, hb, ha, hs0, bidi=wl.bidi, recurrent=recurrent, o=ho,
                                   state_out=hso, stream=e2e_streams[n % 2])

    e2e_steps = max(2, min(args.steps, 6))
    e2e_step(0)
    e2e_step(1)
    torch.cuda.synchronize()
    gdn_device_status(stream)
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_streams[1].wait_event(e0)
    for n in range(e2e_steps):
        e2e_step(n)
    joined = torch.cuda.Event()
    joined.record(e2e_streams[1])
    stream.wait_event(joined)
    e1.record(stream)
    torch.cuda.synchronize()
    gdn_device_status(stream)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world)
    nbytes = lambda *ts: sum(t.numel() * t.element_size() for t in ts if t is not None)

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": wl.dtype, "data": "synthetic",
            "config": workload_config(wl, world),
            "kernel": ("recurrent" if recurrent else
                       "chunk_tc, fp8 E4M3 inputs (dequantising pre-pass)" if fp8_prepass else
                       "chunkwise, pooled, fp8 E4M3 inputs widened to bf16 in shared memory" if args.fp8 else
                       "chunk_tc, normalised read-out (z state, second pass)" if args.normalized else
                       f"chunk_tc, frame-block read-out, blocks of {args.block}" if args.block > 0 else
                       f"chunk_tc, segment-parallel x{args.segments}" if segmented else
                       "chunkwise, single CTA per (dv slice, scan)" if args.kernel == "single" or wl.dv != 128 else
                       "chunkwise, pooled: a state-chain CTA per scan beside preparation workers on the other SMs"),
            "e2e": {"value": world * wl.token_heads / (e2e_ms * 1e-3), "unit": UNIT,
                    "h2d_bytes_per_step": nbytes(hq, hk, hv, hb, ha, hs0,
                                                 *((hsq, hsk, hsv) if args.fp8 else ())),
                    "d2h_bytes_per_step": nbytes(hos[0], hsos[0]),
                    "calls": ("synchronous, one stream" if segmented or rollout or args.fp8 else
                              "gdn_forward_host_async on two alternating streams (2 calls in flight)")},
            "gpu_launches": int(launches),
            "roofline": roofline,
            "clocks": clk.summary()}
    if args.plain_launch:
        line["kernel"] += " (plain launch, for profiling)"
    if rank == 0:
        try:
            line["parity"] = sampled_parity(args, wl, inp, o, s_out,
                                            fp8=(q8, k8, v8, sq, sk, sv) if args.fp8 else None)
        except Exception as e:   # reported, never a reason to lose the line
            line["parity"] = {"checked": False, "error": repr(e)[:300]}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_sample_throughput(wl, inp, target_s=args.ref_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="bidi_720p")
    ap.add_argument("--impl", default="gdn", choices=["gdn", "reference"])
    ap.add_argument("--recurrent", action="store_true",
                    help="time the token-by-token SIMT kernel instead of the chunkwise one")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--fp8", action="store_true",
                    help="fp8 (E4M3) q, k, v with per-head scales (widened in-kernel for dv = 128)")
    ap.add_argument("--normalized", action="store_true",
                    help="normalised read-out with a z state (eps 1e-6)")
    ap.add_argument("--block", type=int, default=0,
                    help="causal workloads: frame-block read-out with blocks of this many tokens")
    ap.add_argument("--segments", type=int, default=0,
                    help="causal workloads: run the segment-parallel scan with this many segments")
    ap.add_argument("--kernel", default="auto", choices=["auto", "single"],
                    help="bf16 chunkwise kernel: by shape (default: the pooled kernel for dk = dv = 128), "
                         "or the single-CTA one for every shape")
    ap.add_argument("--plain-launch", action="store_true",
                    help="launch the pooled kernel without the cooperative attribute (same grid), "
                         "for profilers that replay one launch at a time")
    ap.add_argument("--ref-seconds", type=float, default=None,
                    help="seconds of CPU work per oracle sample (default 15; 8 for --impl reference)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.ref_seconds is None:
        args.ref_seconds = 8.0 if args.impl == "reference" else 15.0
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        return run_reference(args, world, rank)
    world, rank, local = dist_setup()
    try:
        return run_gpu(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
