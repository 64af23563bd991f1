"""Throughput of libmxq's block-scaled quantization on B200.

Headline workload: online layer-by-layer conversion of a 36-layer bf16 decoder
weight stack to MXFP6 E2M3 and to AXS-6 (per layer q 4096x2560, k and v
1024x2560, o 2560x4096, gate and up 9728x2560, down 2560x9728, stored
[out, in] so the blocks of 32 run along the input dim; N(0, 0.02), drawn on the
device from seeded generators). One step = the whole stack converted to both
formats, one layer at a time: for each layer l one grouped launch
(mxq_quantize_grouped, the layer's seven tensors) to E2M3 and one to AXS-6 of
layer (l + 18) mod 36, 72 launches. Each launch reads a 202 MB layer (above the
126 MB L2) last read 18 layers (about 10 GB of traffic) earlier.
Metric: algorithmic bytes moved (values in + packed codes + scales) / device
time, GB/s, and the fraction of the measured HBM copy peak.

Timing: the step is one CUDA graph (72 kernel nodes, nothing between them),
uploaded to the device first (cudaGraphUpload), then replayed K times between
CUDA events on the launching stream; clocks and throttle reasons are sampled
through NVML (the CUDA device found by its UUID) while it runs, and a region
that saw a thermal or hardware slowdown, or a clock stuck well below the
maximum with no reason given, is taken once more (all ranks alike; the dropped
one is listed under clocks.rejected_runs). The device status word is checked
after every timed region: a kernel whose bounded wait ran out leaves partial
outputs, and then no speed is reported. The roofline's kernel is the grouped
quantize (its E2M3 and AXS-6 instances): the timed region launches nothing
else. per_format: each format's 36 launches alone. e2e: one layer per step
through the public Python API from pinned host memory, the host->device copy
of its weights and the device->host copy of both formats' codes and scales
inside the timed region. cpu_baseline: the CPU oracle on row slices of the same
workload (the workload's own bits, from the counter-based generator), on all
host threads (and on one, under single_thread). workloads: every other
workload's ops, each timed alone, including the bf16 4096x4096 weight step
(MXFP6 E2M3 + E3M2 quantize + dequantize in one batch launch).

    python bench.py [--gpus N --steps K --warmup W] [--impl reference] [--no-workloads]
Multi-GPU (torchrun): independent replicas, one per GPU, no collective on the
data path; value = all ranks' bytes / max over ranks of the device time.
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

import synthetic  # noqa: E402

METRIC = "quantize/fake-quant GB/s (bytes in+out) and % of B200 HBM peak, per format"
WORKLOAD = ("online layer-by-layer conversion of a 36-layer bf16 decoder weight stack (per layer q 4096x2560, "
            "k 1024x2560, v 1024x2560, o 2560x4096, gate 9728x2560, up 9728x2560, down 2560x9728, [out, in], "
            "N(0,0.02), seed 2) to MXFP6 E2M3 and to AXS-6, blocks of 32 along the input dim")
WEIGHT_WORKLOAD = "mxfp6_e2m3+e3m2 quantize+dequantize, bf16 4096x4096 weight N(0,0.02) with 0.1% outliers x50, seed 1"
STACK_FORMATS = ("mxfp6_e2m3", "axs6")
FALLBACK_HBM = 6650.0
NOMINAL_HBM = 8000.0  # B200 HBM3e, nominal GB/s (context only; fractions are of the measured copy peak)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM, "fallback"


def sources_sha256(names):
    """sha256 over the named files of the kernel sources (name + contents, in the given order)."""
    import hashlib
    csrc = os.path.join(ROOT, "block_scaled_microscaling_b200", "csrc")
    h = hashlib.sha256()
    for nm in names:
        h.update(nm.encode())
        with open(os.path.join(csrc, nm), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def ncu_traffic(kernel):
    """DRAM bytes per launch of `kernel` from the committed ncu capture, or None when the
    kernel's source files have changed since that capture (or it was not captured)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        e = json.load(f).get("kernels", {}).get(kernel)
    if not e:
        return None
    try:
        if sources_sha256(e["sources"]) != e["sources_sha256"]:
            return None
    except OSError:
        return None
    return int(e["bytes_per_launch"])


def nbytes_q(fmt, n_elems, in_bytes):
    """Algorithmic bytes of one quantize (or dequantize) of n_elems values."""
    bits = {"axs6": 6, "mxfp6_e2m3": 6, "mxfp6_e3m2": 6, "mxfp8": 8, "mxfp4": 4}[fmt]
    sb = 2 if fmt == "axs6" else 1
    return n_elems * in_bytes + n_elems * bits // 8 + n_elems // 32 * sb


# ---- clocks ---------------------------------------------------------------------------

class ClockSampler:
    """SM clock and clock-event reasons of one GPU, sampled by NVML every `period` s."""
    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    # a timed region that saw one of these is not kept
    REJECT = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")

    def __init__(self, index, period=0.002, uuid=None):
        self.samples = []
        self.period = period
        self.ok = False
        self.match = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h, self.match = self.handle(pynvml, index, uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report it, never guess
            self.err = str(e)
        self._stop = threading.Event()

    @staticmethod
    def handle(nv, index, uuid):
        """NVML numbers every GPU of the machine, CUDA only the visible ones: find the CUDA
        device by its UUID, and by index only when that fails."""
        if uuid:
            u = str(uuid)
            try:
                return nv.nvmlDeviceGetHandleByUUID(u if u.startswith("GPU-") else "GPU-" + u), "uuid"
            except Exception:
                pass
        return nv.nvmlDeviceGetHandleByIndex(index), "index"

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()
            # one sample right at the end of the region as well
            try:
                self.samples.append((self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM),
                                     self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)))
            except Exception:
                pass

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        mhz = [m for m, _ in self.samples] or [None]
        seen = set()
        for _, r in self.samples:
            for name, bit in self.REASONS.items():
                if r & bit:
                    seen.add(name)
        return {"sm_mhz": statistics.median(mhz) if mhz[0] is not None else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(seen), "samples": len(self.samples), "nvml_device": self.match}

    @classmethod
    def rejected(cls, summary):
        """True for a region that saw a thermal or hardware slowdown, or whose median SM clock
        sat well below the maximum with no reason given (a clock lock left by someone else)."""
        reasons = summary.get("reasons") or []
        if any(r in cls.REJECT for r in reasons):
            return True
        mhz, top = summary.get("sm_mhz"), summary.get("sm_max_mhz")
        return bool(mhz and top and mhz < 0.9 * top and not reasons)


# ---- the oracle as CPU baseline / reference arm -----------------------------------------

def cpu_threads():
    """Host threads for the oracle timing: the cores this process may run on (at most 32)."""
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count() or 1
    return max(1, min(n, 32))


def oracle_pool(n_slices=24, rows=32, seed=2):
    """Row slices of the decoder stack with the workload's own bits: for each slice a random
    (layer, tensor, first row), its rows drawn from the counter-based generator at their element
    offsets. Made once, before any timing."""
    rng = np.random.default_rng(12345)
    pool = []
    for _ in range(n_slices):
        layer = int(rng.integers(synthetic.N_LAYERS))
        k = int(rng.integers(len(synthetic.DECODER_LAYER)))
        _, nrows, cols = synthetic.DECODER_LAYER[k]
        r0 = int(rng.integers(nrows - rows + 1))
        v = synthetic.normals(seed, layer * 7 + k, rows * cols, start=r0 * cols) * 0.02
        pool.append(synthetic.f32_to_bf16_bits(synthetic.to_f32(v)).reshape(rows, cols))
    return pool


def oracle_throughput(pool, budget_s=10.0, threads=1, formats=STACK_FORMATS):
    """The CPU oracle quantizing the slices of `pool` (bf16 bits) to each of `formats`, round
    robin, for about budget_s seconds on `threads` host threads at once: the oracle's C calls
    release the GIL and keep no shared state, each thread takes its own slices. Returns
    (GB/s of algorithmic bytes over all threads, info)."""
    import oracle
    oracle.lib()  # load once, before the threads start
    done = [0] * threads
    count = [0] * threads
    elems = [0] * threads
    t0 = time.perf_counter()

    def work(k):
        i = k
        while True:
            xs = pool[i % len(pool)]
            for fmt in formats:
                oracle.quantize(xs, fmt)
                done[k] += nbytes_q(fmt, xs.size, 2)
            count[k] += 1
            elems[k] += xs.size
            i += threads
            if time.perf_counter() - t0 >= budget_s:
                break

    if threads == 1:
        work(0)
    else:
        ts = [threading.Thread(target=work, args=(k,)) for k in range(threads)]
        for t in ts:
            t.start()
        for t in ts:
            t.join()
    el = time.perf_counter() - t0
    return sum(done) / el / 1e9, {"samples": sum(count), "seconds": round(el, 2), "elements": int(sum(elems)),
                                  "threads": threads}


def stack_step_bytes():
    """Algorithmic bytes of one step: the whole stack quantized to both formats."""
    n = sum(r * c for _, r, c in synthetic.DECODER_LAYER) * synthetic.N_LAYERS
    return sum(nbytes_q(f, n, 2) for f in STACK_FORMATS), n


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    pool = oracle_pool()
    nt = cpu_threads()
    per_step = []
    for _ in range(args.warmup):
        oracle_throughput(pool, budget_s=0.2, threads=nt)
    for _ in range(args.steps):
        v, info = oracle_throughput(pool, budget_s=max(0.2, args.ref_seconds / max(1, args.steps)), threads=nt)
        per_step.append(v)
    value = statistics.mean(per_step)
    step_bytes, _ = stack_step_bytes()
    sample = (f"{len(pool)} slices of 32 rows of the stack's tensors (the workload's own bits), each quantized "
              f"to MXFP6 E2M3 and AXS-6, oracle in C on {nt} host threads, ~{args.ref_seconds:.0f} s in total")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_bytes / (value * 1e9) * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "sample": sample},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": nt, "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---- multi-rank host logic (replicas; no data-path collective) ---------------------------

def max_over_ranks(value, dist, device):
    """The largest `value` over all ranks (timing only); identity on one process."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_gbs(world, bytes_per_step, steps, ms_total_max):
    """Whole-job throughput: every rank moved bytes_per_step * steps; time = slowest rank."""
    return world * bytes_per_step * steps / (ms_total_max * 1e-3) / 1e9


def timed_replay(torch, graph, device, dist, sampler, attempts=2, replays=1, after=None):
    """Device time (ms) of `replays` back-to-back replays of `graph` between CUDA events on the
    current stream, with the clocks sampled while they run. A region whose clock record is
    rejected (ClockSampler.rejected) on any rank is taken again, up to `attempts` in all; every
    rank takes the same number, since the decision is a max over ranks. `after` (if given) runs
    once each region has synchronized (the device status check). Returns (ms, clocks) of the
    last region; clocks lists the rejected ones under "rejected_runs"."""
    multi = dist is not None and dist.is_initialized() and dist.get_world_size() > 1
    rejected = []
    for attempt in range(attempts):
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        if multi:
            dist.barrier()
        torch.cuda.synchronize()
        with sampler() as clk:
            start.record()
            for _ in range(replays):
                graph.replay()
            end.record()
            torch.cuda.synchronize()
        if after is not None:
            after()
        if multi:
            dist.barrier()
        ms, clocks = start.elapsed_time(end), clk.summary()
        mine = ClockSampler.rejected(clocks)
        bad = max_over_ranks(1.0 if mine else 0.0, dist if multi else None, device)
        if bad == 0.0 or attempt == attempts - 1:
            if rejected:
                clocks["rejected_runs"] = rejected
            return ms, clocks
        rejected.append({"ms": round(ms, 4), "clocks": clocks, "on": "this rank" if mine else "another rank"})


# ---- the GPU arm --------------------------------------------------------------------------

def make_sets(torch, mxq, w_dev, nsets):
    sets = []
    for _ in range(nsets):
        x = w_dev.clone()
        s = {"x": x}
        for fmt, tag in (("mxfp6_e2m3", "a"), ("mxfp6_e3m2", "b")):
            c, sc = mxq.quantize(x, fmt)
            s["c" + tag], s["s" + tag] = c, sc
            s["y" + tag] = torch.empty_like(x)
        sets.append(s)
    return sets


def step_ops(mxq, sets, k):
    """The four launches of step k, each reading a buffer set last touched >= 4 steps ago."""
    n = len(sets)
    i = k % n
    a, b, c, d = sets[i], sets[(i + 4) % n], sets[(i + 2) % n], sets[(i + 6) % n]
    return [
        ("quantize_e2m3", lambda: mxq.quantize(a["x"], "mxfp6_e2m3", codes=a["ca"], scales=a["sa"])),
        ("quantize_e3m2", lambda: mxq.quantize(b["x"], "mxfp6_e3m2", codes=b["cb"], scales=b["sb"])),
        ("dequantize_e2m3", lambda: mxq.dequantize(c["ca"], c["sa"], "mxfp6_e2m3", c["x"].shape, out=c["ya"])),
        ("dequantize_e3m2", lambda: mxq.dequantize(d["cb"], d["sb"], "mxfp6_e3m2", d["x"].shape, out=d["yb"])),
    ]


def step_batch(mxq, sets, k):
    """Step k as one launch: the same four conversions through the batch entry point."""
    n = len(sets)
    i = k % n
    a, b, c, d = sets[i], sets[(i + 4) % n], sets[(i + 2) % n], sets[(i + 6) % n]
    ops = [("quantize", "mxfp6_e2m3", a["x"], a["ca"], a["sa"]),
           ("quantize", "mxfp6_e3m2", b["x"], b["cb"], b["sb"]),
           ("dequantize", "mxfp6_e2m3", c["ca"], c["sa"], c["ya"]),
           ("dequantize", "mxfp6_e3m2", d["cb"], d["sb"], d["yb"])]
    return lambda: mxq.batch(ops)


def decoder_stack(torch, seed=2):
    """The 36 layers of seven bf16 [out, in] weights, N(0, 0.02), drawn on the device from a
    seeded generator (the host generator's bits would take minutes at 3.6G values; parity on
    those bits is a test)."""
    dev = torch.device("cuda")
    gen = torch.Generator(device=dev)
    layers = []
    for l in range(synthetic.N_LAYERS):
        gen.manual_seed(seed * 1000 + l)
        layers.append([(torch.randn(r, c, device=dev, generator=gen) * 0.02).to(torch.bfloat16)
                       for _, r, c in synthetic.DECODER_LAYER])
    return layers


def stack_step(mxq, layers, outs):
    """The 72 launches of one step: layer l to E2M3, then layer (l + 18) mod 36 to AXS-6, for
    l = 0..35, so each launch reads a layer last read 18 layers earlier. outs[fmt][l] holds
    layer l's preallocated codes and scales."""
    L = len(layers)
    fns = []
    for l in range(L):
        for fmt, j in ((STACK_FORMATS[0], l), (STACK_FORMATS[1], (l + L // 2) % L)):
            fns.append(lambda ws=layers[j], o=outs[fmt][j], f=fmt: mxq.quantize_grouped(ws, f, outs=o))
    return fns


def graph_of(torch, fns):
    """One CUDA graph that launches every callable of `fns` in order on one stream."""
    g = torch.cuda.CUDAGraph()
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g, stream=stream):
            for fn in fns:
                fn()
    torch.cuda.current_stream().wait_stream(stream)
    return g


def upload_graph(torch, g):
    """Upload an instantiated graph to the device before its first replay. Otherwise that one-time
    setup (about 5 us per step for a graph of K steps) lands inside the first replay, which is the
    timed one. Returns whether the upload ran."""
    try:
        from cuda.bindings import runtime as rt
    except ImportError:
        return False
    (err,) = rt.cudaGraphUpload(g.raw_cuda_graph_exec(), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return err == rt.cudaError_t.cudaSuccess


def time_graph(torch, g, replays=1):
    """Device time (ms) of `replays` back-to-back replays, CUDA events on the launching stream."""
    g.replay()
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(replays):
        g.replay()
    end.record()
    torch.cuda.synchronize()
    return start.elapsed_time(end)


def e2e_measure(torch, mxq, steps):
    """Public API from pinned host memory, one layer per step: the host->device copy of the
    layer's seven weights, its grouped conversions to E2M3 and to AXS-6, the device->host copy
    of both formats' codes and scales. The host->device copy of step k+1 runs on its own stream
    and overlaps the device->host copies of step k (PCIe is full duplex); two device buffer sets
    alternate, fed from two distinct pinned host layers."""
    dev = torch.device("cuda")
    gen = torch.Generator()
    host = []
    for h in range(2):
        gen.manual_seed(2 * 1000 + h)
        host.append([(torch.randn(r, c, generator=gen) * 0.02).to(torch.bfloat16).pin_memory()
                     for _, r, c in synthetic.DECODER_LAYER])
    sets = []
    for _ in range(2):
        xs = [torch.empty_like(t, device=dev) for t in host[0]]
        sets.append({"x": xs, "out": {f: mxq.quantize_grouped(xs, f) for f in STACK_FORMATS}})
    outs_h = {f: [(torch.empty_like(c, device="cpu").pin_memory(), torch.empty_like(s, device="cpu").pin_memory())
                  for c, s in sets[0]["out"][f]] for f in STACK_FORMATS}
    h2d = sum(t.numel() * t.element_size() for t in host[0])
    d2h = sum(c.numel() * c.element_size() + s.numel() * s.element_size() for f in STACK_FORMATS for c, s in outs_h[f])
    s_in, s_work = torch.cuda.Stream(), torch.cuda.Stream()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    done = [None, None]  # event after the conversions that last read set p's inputs
    torch.cuda.synchronize()
    for it in range(steps + 2):
        if it == 2:
            s_in.synchronize()
            s_work.synchronize()
            t0.record(s_in)
        p = it % 2
        cur = sets[p]
        with torch.cuda.stream(s_in):
            if done[p] is not None:
                s_in.wait_event(done[p])
            for d, h in zip(cur["x"], host[it % 2]):
                d.copy_(h, non_blocking=True)
            arrived = torch.cuda.Event()
            arrived.record(s_in)
        with torch.cuda.stream(s_work):
            s_work.wait_event(arrived)
            for f in STACK_FORMATS:
                mxq.quantize_grouped(cur["x"], f, outs=cur["out"][f])
            done[p] = torch.cuda.Event()
            done[p].record(s_work)
            for f in STACK_FORMATS:
                for (c, s), (hc, hs) in zip(cur["out"][f], outs_h[f]):
                    hc.copy_(c, non_blocking=True)
                    hs.copy_(s, non_blocking=True)
    t1.record(s_work)
    torch.cuda.synchronize()
    mxq.check_device()
    ms = t0.elapsed_time(t1) / steps
    n = sum(t.numel() for t in host[0])
    step_bytes = sum(nbytes_q(f, n, 2) for f in STACK_FORMATS)
    return {"value": round(step_bytes / (ms * 1e-3) / 1e9, 2), "unit": "GB/s", "ms_per_step": round(ms, 4),
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "step": "one decoder layer: H2D of its 7 weights, grouped quantize to E2M3 and to AXS-6, D2H of both "
                    "formats' codes and scales",
            "overlap": "H2D of step k+1 on its own stream during the D2H of step k"}


def time_launches(torch, fns, reps):
    """Mean device time of each callable: a graph of `reps` back-to-back launches of it, timed as a whole."""
    out = []
    for fn in fns:
        g = graph_of(torch, [fn] * reps)
        out.append(time_graph(torch, g) / reps)
        del g
    return out


def workloads_breakdown(torch, mxq, hbm):
    """Device GB/s of the ops of the other workloads (each launch reads HBM-resident data:
    tensors above L2 size, or rotated copies; the 128x256 quick start is latency-bound)."""
    dev = torch.device("cuda")
    gen = torch.Generator(device=dev)
    out = {}

    def rec(name, b, n, ms):
        gbs = b / (ms * 1e-3) / 1e9
        out[name] = {"ms": round(ms, 4), "GB/s": round(gbs, 1), "Gelem/s": round(n / (ms * 1e-3) / 1e9, 1),
                     "frac_hbm": round(gbs / hbm, 4), "frac_nominal": round(gbs / NOMINAL_HBM, 4), "bytes": int(b)}

    # 1: AXS-6 quick-start fp32 128x256 (L2-resident, launch-latency bound)
    x1 = torch.randn(128, 256, device=dev, generator=gen.manual_seed(0))
    o1 = torch.empty_like(x1)
    c1, s1 = mxq.quantize(x1, "axs6")
    t = time_launches(torch, [lambda: mxq.fake_quantize(x1, "axs6", out=o1), lambda: mxq.quantize(x1, "axs6", codes=c1, scales=s1),
                              lambda: mxq.dequantize(c1, s1, "axs6", x1.shape, out=o1)], 50)
    n1 = x1.numel()
    rec("c1_axs6_fake_quantize_f32", 8 * n1, n1, t[0])
    rec("c1_axs6_quantize_f32", nbytes_q("axs6", n1, 4), n1, t[1])
    rec("c1_axs6_dequantize_f32", nbytes_q("axs6", n1, 4), n1, t[2])

    # 2: the bf16 4096x4096 weight: one step = MXFP6 E2M3 + E3M2 quantize + dequantize in one batch
    # launch, 8 rotating buffer sets (~1 GB: every launch reads data last touched >= 4 steps
    # earlier); per_op: the four single-operation kernels, each a graph of 400 launches of it alone
    w_host, _ = synthetic.weight_with_outliers(seed=1)
    w = torch.from_numpy(w_host.view(np.int16)).view(torch.bfloat16).cuda()
    sets = make_sets(torch, mxq, w, 8)
    n2 = w.numel()
    op_bytes = nbytes_q("mxfp6_e2m3", n2, 2)
    K2 = 400
    g = graph_of(torch, [step_batch(mxq, sets, k) for k in range(K2)])
    upload_graph(torch, g)
    ms = time_graph(torch, g) / K2
    del g
    rec("c2_weight_batch_step_bf16", 4 * op_bytes, 4 * n2, ms)
    out["c2_weight_batch_step_bf16"]["launches"] = "one mxq_run_batch launch per step (the four conversions)"
    for j, nm in enumerate([nm for nm, _ in step_ops(mxq, sets, 0)]):
        g = graph_of(torch, [step_ops(mxq, sets, k)[j][1] for k in range(K2)])
        ms = time_graph(torch, g) / K2
        del g
        rec(f"c2_weight_{nm}_bf16", op_bytes, n2, ms)
    # column-direction blocks of the same weight (32 rows of a column), transposed layout: 8 launches
    # per round on the 8 sets, so each reads data last touched 7 launches (330 MB) earlier; 50
    # rounds, 400 launches per graph as for the single-operation rows
    ccs = [mxq.quantize_cols(st["x"], "mxfp6_e2m3") for st in sets]
    ts = time_launches(torch, [
        lambda: [mxq.quantize_cols(st["x"], "mxfp6_e2m3", codes=c, scales=sc_) for st, (c, sc_) in zip(sets, ccs)],
        lambda: [mxq.dequantize_cols(c, sc_, "mxfp6_e2m3", st["x"].shape, out=st["ya"])
                 for st, (c, sc_) in zip(sets, ccs)]], 50)
    rec("c2_weight_quantize_cols_e2m3_bf16", op_bytes, n2, ts[0] / len(sets))
    rec("c2_weight_dequantize_cols_e2m3_bf16", op_bytes, n2, ts[1] / len(sets))
    del sets, ccs, w
    torch.cuda.empty_cache()
    mxq.check_device()

    # 4: activations bf16 16384x8192 (0.5*t3, 16 channels x100), gradients fp32 N(0,1e-3)
    gen.manual_seed(3)
    z = torch.randn(4, 16384, 8192, device=dev, generator=gen)
    a = (0.5 * z[0] / torch.sqrt((z[1] ** 2 + z[2] ** 2 + z[3] ** 2) / 3))
    a[:, synthetic.outlier_channels()] *= 100
    a = a.to(torch.bfloat16)
    del z
    g = torch.randn(16384, 8192, device=dev, generator=gen) * 1e-3
    go = torch.empty_like(g)
    for fmt in ("mxfp8", "mxfp6_e2m3"):
        c, s = mxq.quantize(a, fmt)
        y = torch.empty_like(a)
        ts = time_launches(torch, [lambda: mxq.quantize(a, fmt, codes=c, scales=s),
                                   lambda: mxq.dequantize(c, s, fmt, a.shape, out=y)], 10)
        rec(f"c4_act_{fmt}_quantize_bf16", nbytes_q(fmt, a.numel(), 2), a.numel(), ts[0])
        rec(f"c4_act_{fmt}_dequantize_bf16", nbytes_q(fmt, a.numel(), 2), a.numel(), ts[1])
        del c, s, y
    ts = time_launches(torch, [lambda: mxq.fake_quantize(g, "axs6", out=go)], 10)
    rec("c4_grad_axs6_fake_quantize_f32", 8 * g.numel(), g.numel(), ts[0])
    # column-direction blocks of the activations (the backward pass's K-contiguous operand)
    cc, cs = mxq.quantize_cols(a, "mxfp6_e2m3")
    y = torch.empty_like(a)
    ts = time_launches(torch, [lambda: mxq.quantize_cols(a, "mxfp6_e2m3", codes=cc, scales=cs),
                               lambda: mxq.dequantize_cols(cc, cs, "mxfp6_e2m3", a.shape, out=y)], 10)
    rec("c4_act_quantize_cols_e2m3_bf16", nbytes_q("mxfp6_e2m3", a.numel(), 2), a.numel(), ts[0])
    rec("c4_act_dequantize_cols_e2m3_bf16", nbytes_q("mxfp6_e2m3", a.numel(), 2), a.numel(), ts[1])
    del a, g, go, cc, cs, y
    mxq.check_device()
    torch.cuda.empty_cache()

    # 5: scores fp32 4096 x 32768 N(0,3) -> exp -> MXFP4
    gen.manual_seed(4)
    sc = torch.randn(4096, 32768, device=dev, generator=gen) * 3
    c5, s5 = mxq.exp_quantize(sc, "mxfp4")
    ts = time_launches(torch, [lambda: mxq.exp_quantize(sc, "mxfp4", codes=c5, scales=s5),
                               lambda: mxq.exp_free_quantize(sc, codes=c5, scales=s5)], 10)
    rec("c5_scores_exp_mxfp4_f32", nbytes_q("mxfp4", sc.numel(), 4), sc.numel(), ts[0])
    # the same stage by the exp-free rule (no exponential), same bytes
    rec("c5_scores_exp_free_mxfp4_f32", nbytes_q("mxfp4", sc.numel(), 4), sc.numel(), ts[1])
    for fmt in ("mxfp6_e2m3", "axs6"):
        c6, s6 = mxq.exp_quantize(sc, fmt)
        ts = time_launches(torch, [lambda: mxq.exp_quantize(sc, fmt, codes=c6, scales=s6)], 10)
        rec(f"c5_scores_exp_{fmt}_f32", nbytes_q(fmt, sc.numel(), 4), sc.numel(), ts[0])
        del c6, s6
    del sc, c5, s5
    mxq.check_device()
    torch.cuda.empty_cache()
    return out


PROFILE_CASES = ["batch_weight", "q_e2m3_weight", "q_e3m2_weight", "dq_e2m3_weight", "q_mxfp8_act", "dq_mxfp8_act", "q_axs6_layer",
                 "q_e2m3_layer", "fq_axs6_grad", "exp_mxfp4_scores", "expfree_mxfp4_scores", "qcols_e2m3_weight",
                 "dqcols_e2m3_weight", "qcols_e2m3_act", "dqcols_e2m3_act", "exmy_e3m3_act", "dq_exmy_e3m3_act",
                 "fq_exmy_e3m3_act", "qmma_mxfp8_act", "dq_e2m3_act", "fq_axs6_quickstart",
                 "swizzle_scales_act", "exp_e2m3_scores", "exp_axs6_scores", "dqcols_e2m3_f32", "stack_steady"]


def profile_case(name, reps):
    """Run one kernel `reps` times on its workload (for ncu captures); prints one line."""
    import torch
    from block_scaled_microscaling_b200 import mxq
    dev = torch.device("cuda")
    gen = torch.Generator(device=dev).manual_seed(0)
    if name == "batch_weight":  # one headline step: four conversions on four distinct buffer groups
        w_host, _ = synthetic.weight_with_outliers(seed=1)
        w = torch.from_numpy(w_host.view(np.int16)).view(torch.bfloat16).cuda()
        sets = make_sets(torch, mxq, w, 8)
        fn = step_batch(mxq, sets, 0)
    elif name in ("q_e2m3_weight", "q_e3m2_weight", "dq_e2m3_weight", "qcols_e2m3_weight", "dqcols_e2m3_weight"):
        w_host, _ = synthetic.weight_with_outliers(seed=1)
        x = torch.from_numpy(w_host.view(np.int16)).view(torch.bfloat16).cuda()
        f = "mxfp6_e3m2" if "e3m2" in name else "mxfp6_e2m3"
        c, s = mxq.quantize(x, f)
        y = torch.empty_like(x)
        if name.startswith("qcols"):
            fn = lambda: mxq.quantize_cols(x, f, codes=c, scales=s)
        elif name.startswith("dqcols"):
            cc, cs = mxq.quantize_cols(x, f)
            fn = lambda: mxq.dequantize_cols(cc, cs, f, x.shape, out=y)
        elif name[0] == "q":
            fn = lambda: mxq.quantize(x, f, codes=c, scales=s)
        else:
            fn = lambda: mxq.dequantize(c, s, f, x.shape, out=y)
    elif name in ("qcols_e2m3_act", "dqcols_e2m3_act"):
        x = (torch.randn(16384, 8192, device=dev, generator=gen) * 0.5).to(torch.bfloat16)
        cc, cs = mxq.quantize_cols(x, "mxfp6_e2m3")
        y = torch.empty_like(x)
        fn = (lambda: mxq.quantize_cols(x, "mxfp6_e2m3", codes=cc, scales=cs)) if name[0] == "q" else \
            (lambda: mxq.dequantize_cols(cc, cs, "mxfp6_e2m3", x.shape, out=y))
    elif name == "dqcols_e2m3_f32":
        x = torch.randn(8192, 8192, device=dev, generator=gen) * 0.02
        cc, cs = mxq.quantize_cols(x, "mxfp6_e2m3")
        y = torch.empty_like(x)
        fn = lambda: mxq.dequantize_cols(cc, cs, "mxfp6_e2m3", x.shape, out=y)
    elif name == "dq_e2m3_act":
        x = (torch.randn(16384, 8192, device=dev, generator=gen) * 0.5).to(torch.bfloat16)
        c, s = mxq.quantize(x, "mxfp6_e2m3")
        y = torch.empty_like(x)
        fn = lambda: mxq.dequantize(c, s, "mxfp6_e2m3", x.shape, out=y)
    elif name == "fq_axs6_quickstart":
        x = torch.randn(128, 256, device=dev, generator=gen)
        o = torch.empty_like(x)
        fn = lambda: mxq.fake_quantize(x, "axs6", out=o)
    elif name == "swizzle_scales_act":
        x = (torch.randn(16384, 8192, device=dev, generator=gen) * 0.5).to(torch.bfloat16)
        _, s = mxq.quantize(x, "mxfp8")
        o = mxq.swizzle_scales(s)
        fn = lambda: mxq.swizzle_scales(s, out=o)
    elif name in ("exp_e2m3_scores", "exp_axs6_scores"):
        fmt = "mxfp6_e2m3" if "e2m3" in name else "axs6"
        sc = torch.randn(4096, 32768, device=dev, generator=gen) * 3
        c, s = mxq.exp_quantize(sc, fmt)
        fn = lambda: mxq.exp_quantize(sc, fmt, codes=c, scales=s)
    elif name in ("exmy_e3m3_act", "dq_exmy_e3m3_act", "fq_exmy_e3m3_act"):
        x = (torch.randn(16384, 8192, device=dev, generator=gen) * 0.5).to(torch.bfloat16)
        c, s = mxq.quantize_exmy(x, 3, 3)
        y = torch.empty_like(x)
        if name == "exmy_e3m3_act":
            fn = lambda: mxq.quantize_exmy(x, 3, 3, codes=c, scales=s)
        elif name == "dq_exmy_e3m3_act":
            fn = lambda: mxq.dequantize_exmy(c, s, 3, 3, x.shape, out=y)
        else:
            fn = lambda: mxq.fake_quantize_exmy(x, 3, 3, out=y)
    elif name == "qmma_mxfp8_act":
        x = (torch.randn(16384, 8192, device=dev, generator=gen) * 0.5).to(torch.bfloat16)
        c, s = mxq.quantize_mma(x, "mxfp8")
        fn = lambda: mxq.quantize_mma(x, "mxfp8", codes=c, scales=s)
    elif name in ("q_mxfp8_act", "dq_mxfp8_act"):
        x = (torch.randn(16384, 8192, device=dev, generator=gen) * 0.5).to(torch.bfloat16)
        c, s = mxq.quantize(x, "mxfp8")
        y = torch.empty_like(x)
        fn = (lambda: mxq.quantize(x, "mxfp8", codes=c, scales=s)) if name[0] == "q" else \
            (lambda: mxq.dequantize(c, s, "mxfp8", x.shape, out=y))
    elif name in ("q_axs6_layer", "q_e2m3_layer"):
        fmt = "axs6" if "axs6" in name else "mxfp6_e2m3"
        ws = [(torch.randn(r, c_, device=dev, generator=gen) * 0.02).to(torch.bfloat16)
              for _, r, c_ in synthetic.DECODER_LAYER]
        outs = mxq.quantize_grouped(ws, fmt)
        fn = lambda: mxq.quantize_grouped(ws, fmt, outs=outs)
    elif name == "stack_steady":
        # three decoder layers; launch k converts layer k mod 3 to E2M3 (k even) or AXS-6 (k odd),
        # so every launch reads a layer last read three launches (about 850 MB of traffic) earlier
        # and the previous launch's outputs leave L2 during it, as in the timed step: the DRAM
        # counters of one launch then hold its whole traffic (no flush between launches)
        layers = [[(torch.randn(r, c_, device=dev, generator=gen) * 0.02).to(torch.bfloat16)
                   for _, r, c_ in synthetic.DECODER_LAYER] for _ in range(3)]
        outs = {f: [mxq.quantize_grouped(ws, f) for ws in layers] for f in STACK_FORMATS}
        k = [0]

        def fn():
            f = STACK_FORMATS[k[0] % 2]
            mxq.quantize_grouped(layers[k[0] % 3], f, outs=outs[f][k[0] % 3])
            k[0] += 1
    elif name == "fq_axs6_grad":
        g = torch.randn(16384, 8192, device=dev, generator=gen) * 1e-3
        o = torch.empty_like(g)
        fn = lambda: mxq.fake_quantize(g, "axs6", out=o)
    elif name == "exp_mxfp4_scores":
        sc = torch.randn(4096, 32768, device=dev, generator=gen) * 3
        c, s = mxq.exp_quantize(sc, "mxfp4")
        fn = lambda: mxq.exp_quantize(sc, "mxfp4", codes=c, scales=s)
    elif name == "expfree_mxfp4_scores":
        sc = torch.randn(4096, 32768, device=dev, generator=gen) * 3
        c, s = mxq.exp_free_quantize(sc)
        fn = lambda: mxq.exp_free_quantize(sc, codes=c, scales=s)
    else:
        raise SystemExit(f"unknown profile case {name}; one of {PROFILE_CASES}")
    for _ in range(reps):
        fn()
    torch.cuda.synchronize()
    print(json.dumps({"profile_case": name, "reps": reps}))
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--profile-case", choices=PROFILE_CASES, default=None,
                    help="run one kernel a few times on its workload and exit (for ncu captures)")
    ap.add_argument("--profile-reps", type=int, default=3)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="mxq", choices=["mxq", "reference"])
    ap.add_argument("--ref-seconds", type=float, default=20.0)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-workloads", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.profile_case:
        return profile_case(args.profile_case, args.profile_reps)

    import torch
    import torch.distributed as dist
    from block_scaled_microscaling_b200 import mxq

    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    hbm, how = peaks()
    dd = dist if world > 1 else None

    # the stack (7.3 GB bf16) and both formats' outputs (5.8 GB), resident in HBM
    layers = decoder_stack(torch)
    outs = {f: [mxq.quantize_grouped(ws, f) for ws in layers] for f in STACK_FORMATS}
    step = stack_step(mxq, layers, outs)
    step_bytes, n = stack_step_bytes()
    launches_per_step = len(step)

    # warm-up: W eager steps, then the step graph W times
    for _ in range(args.warmup):
        for fn in step:
            fn()
    torch.cuda.synchronize()
    mxq.check_device()
    gt = graph_of(torch, step)
    uploaded = upload_graph(torch, gt)
    for _ in range(args.warmup):
        gt.replay()
    torch.cuda.synchronize()
    # timed region: the step graph replayed K times back to back
    uuid = getattr(torch.cuda.get_device_properties(local), "uuid", None)
    ms_total, clocks = timed_replay(torch, gt, "cuda", dd, lambda: ClockSampler(local, uuid=uuid),
                                    replays=args.steps, after=mxq.check_device)
    del gt
    ms_total = max_over_ranks(ms_total, dd, "cuda")
    # each format's 36 launches alone, for the per-format figures (same layers, same rotation)
    per_format = {}
    for j, f in enumerate(STACK_FORMATS):
        g = graph_of(torch, step[j::2])
        ms = time_graph(torch, g, replays=max(3, min(args.steps, 10))) / max(3, min(args.steps, 10))
        del g
        b = nbytes_q(f, n, 2)
        per_format[f] = {"ms_per_stack": round(ms, 4), "GB/s": round(b / (ms * 1e-3) / 1e9, 1),
                         "Gelem/s": round(n / (ms * 1e-3) / 1e9, 1), "frac_hbm": round(b / (ms * 1e-3) / 1e9 / hbm, 4),
                         "frac_nominal": round(b / (ms * 1e-3) / 1e9 / NOMINAL_HBM, 4), "bytes_per_stack": int(b)}
    mxq.check_device()
    del outs, layers, step
    torch.cuda.empty_cache()

    ms_step = ms_total / args.steps
    value = job_gbs(world, step_bytes, args.steps, ms_total)
    # the timed region launches the grouped quantize kernel only (its E2M3 and AXS-6 instances,
    # 72 launches per step): algorithmic bytes per launch / average launch duration
    bytes_per_launch = step_bytes / launches_per_step
    ach = bytes_per_launch / (ms_step / launches_per_step * 1e-3) / 1e9

    result = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": WORKLOAD, "elements_per_step": 2 * n, "bytes_per_step": step_bytes,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "inputs larger than L2: each launch reads a 202 MB layer last read 18 layers "
                         "(about 10 GB of traffic) earlier",
                   "launches": f"{launches_per_step} mxq_quantize_grouped launches per step: layer l to E2M3, "
                               "layer (l+18) mod 36 to AXS-6, l = 0..35",
                   "timing": "one CUDA graph of one step replayed K times between CUDA events on the launching "
                             "stream" + (", uploaded to the device first" if uploaded else "")
                             + "; the device status word checked after the region"},
        "frac_hbm": round(value / world / hbm, 4),
        "per_format": per_format,
        "gelem_per_s": round(world * 2 * n * args.steps / (ms_total * 1e-3) / 1e9, 2),
        "roofline": {"bound": "hbm", "kernel": "grouped k_quantize<fmt, bf16, 64> (E2M3 and AXS-6 instances)",
                     "achieved": round(ach, 1), "peak": hbm, "peak_source": how, "unit": "GB/s",
                     "frac": round(ach / hbm, 4), "peak_nominal": NOMINAL_HBM,
                     "frac_nominal": round(ach / NOMINAL_HBM, 4), "traffic": ncu_traffic("grouped_layer"),
                     "traffic_source": "DRAM bytes read + written per launch, ncu in the step's steady state "
                                       "(profiles/k_quantize_grouped_decoder_layer_steady_traffic.md)",
                     "algorithmic_bytes_per_launch": int(bytes_per_launch),
                     "launch_ms": round(ms_step / launches_per_step, 5)},
        "clocks": clocks,
        "gpu_launches": launches_per_step * args.steps,
    }
    if rank == 0:
        result["e2e"] = e2e_measure(torch, mxq, steps=max(3, min(args.steps, 12)))
        if not args.no_cpu_baseline:
            pool = oracle_pool()
            v1, i1 = oracle_throughput(pool, budget_s=args.cpu_seconds / 2)
            nt = cpu_threads()
            vn, i_n = oracle_throughput(pool, budget_s=args.cpu_seconds / 2, threads=nt)
            result["cpu_baseline"] = {
                "value": round(vn, 4), "unit": "GB/s", "cores": nt, "kind": "oracle",
                "sample": f"{i_n['samples']} quantizations of 32-row slices of the stack's tensors (the workload's "
                          f"own bits) to MXFP6 E2M3 and AXS-6, {i_n['elements']} values, {i_n['seconds']} s on "
                          f"{nt} threads",
                "single_thread": {"value": round(v1, 4), "cores": 1,
                                  "sample": f"{i1['samples']} slices, {i1['seconds']} s"}}
        if not args.no_workloads:
            result["workloads"] = workloads_breakdown(torch, mxq, hbm)
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
