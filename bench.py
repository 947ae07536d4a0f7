"""Throughput of one MLA paged-decode step on B200, as one JSON line.

A step is the whole hot path over one batch: the metadata kernel, the split-KV
decode kernel and the combine kernel, launched through the C ABI on one
stream.  The headline workload is the compute-bound decode configuration
(64 sequences x 4096 tokens, h_q = 128, one shared 576-wide KV head, 64-token
pages, shuffled page table); its 302 MB cache is larger than the 126 MB L2,
so consecutive steps do not hit in L2.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl reference]

Without ``--workload`` the line also carries ``workloads``: the same
measurement (its own timed region of 200 steps) for the tiny, variable-length
memory-bound, causal MTP and long-context configurations.  Per-kernel device
times come from separate loops of 64 back-to-back launches of one kernel
between two CUDA events, after the timed region, so they never perturb the
step time and never rest on a handful of samples.

``--impl reference`` times the fp64 CPU oracle on this machine's cores on a
bounded sample of the same workload (the pages ship no runnable code).  Under
torchrun each rank runs an independent replica (the path needs no exchange);
``value`` is the work of all ranks over the slowest rank's time.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from mla_paged_kv_get_b200 import inputs  # noqa: E402

WORKLOADS = {inputs.CONFIG_NAMES[i]: i for i in inputs.CONFIG_NAMES}
DEFAULT_WORKLOAD = "compute_bound"
METRIC = "MLA paged decode TFLOPS and HBM GB/s on 1 B200, % of roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def algorithmic_work(w) -> tuple[int, int]:
    """(flops, bytes) the method must spend: valid (row, key) pairs only.

    flops = 2 * (576 + 512) * sum over rows of visible keys; bytes = the cache
    rows read once (V is the same row) + q + out + lse + page-table entries +
    seqlens.  Page-tail rounding and split partials are overhead, not counted.
    """
    hg = w.h_q // w.h_kv
    flops = 0
    nbytes = 0
    for L in w.seqlens.tolist():
        for s in range(w.s_q):
            n = L - (w.s_q - 1 - s) if w.causal else L
            flops += 2 * (576 + 512) * max(0, min(n, L)) * hg * w.h_kv
        nbytes += L * w.h_kv * 576 * 2
        nbytes += w.s_q * w.h_q * (576 * 2 + 512 * 2 + 4)
        nbytes += ((L + 63) // 64) * 4 + 4
    return flops, nbytes


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def load_traffic(workload: str):
    """DRAM bytes per decode launch from the committed ncu summary, if any."""
    path = os.path.join(ROOT, "profiles", f"decode_{workload}_traffic.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d.get("dram_bytes_per_launch"), d.get("kernel_source_sha")
    return None, None


# the files the decode kernels (and the tensor maps they are launched with) are built from
DECODE_SOURCES = ("capi.cu", "decode.cu", "decode.cuh", "decode_pair.cu", "ptx.cuh", "segments.cuh")


def source_sha() -> str:
    """Hash of the decode kernels' sources: stored ncu counters apply only while it is unchanged."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "mla_paged_kv_get_b200", "csrc")
    for name in DECODE_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


class ClockSampler:
    """nvidia-smi clock/throttle samples of one GPU while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.proc = None
        self.lines: list[str] = []
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            sel = ["-i", uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"]
        except Exception:
            sel = []
        self.cmd = ["nvidia-smi", *sel, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                    "-lms", "100"]

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(self.cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for name, val in zip(names, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        import datetime
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def cpu_oracle_timing(w, budget_s: float = 15.0):
    """Time the fp64 oracle, as it stands, on a bounded sample of sequences."""
    import numpy as np
    from oracle import mla_oracle
    try:
        from threadpoolctl import threadpool_info
        cores = max((i.get("num_threads", 1) for i in threadpool_info()), default=os.cpu_count())
    except Exception:
        cores = os.cpu_count()
    q = w.q.float().double().numpy()
    k = w.k_cache.float().double().numpy()
    bt = w.block_table.numpy().astype(np.int64)
    sl = w.seqlens.numpy().astype(np.int64)
    flops_per_b = []
    for b in range(w.batch):
        L = int(sl[b])
        f = 0
        for s in range(w.s_q):
            n = L - (w.s_q - 1 - s) if w.causal else L
            f += 2 * (576 + 512) * max(0, min(n, L)) * w.h_q
        flops_per_b.append(f)
    done_flops, done_bytes, n_done = 0, 0, 0
    t0 = time.perf_counter()
    for b in range(w.batch):
        mla_oracle.decode_dense(q, k, bt, sl, w.h_kv, w.causal, w.scale, batches=[b])
        done_flops += flops_per_b[b]
        done_bytes += int(sl[b]) * w.h_kv * 576 * 2
        n_done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": done_flops / dt / 1e12, "unit": "TFLOP/s", "cores": int(cores), "kind": "oracle",
            "sample": f"fp64 numpy oracle (decode_dense) on {n_done} of {w.batch} sequences of the "
                      f"{w.name} workload, {dt:.1f} s; inputs widened to fp64 before timing",
            "hbm_equiv_gbs": done_bytes / dt / 1e9, "seconds": dt}


def torch_native_timing(w, q, k, bt, sl, flops: int, reps: int = 10):
    """The same decode in plain PyTorch on the GPU, timed next to the kernels.

    Dense page gather through the block table, S = scale * Q.K^T (bf16 matmul), the
    length (and causal) mask, softmax in fp32, O = P.V with V the first 512 columns,
    and the logsumexp.  A same-box comparison on the same algorithmic work, not a
    path the library ever takes.
    """
    B, s_q, h_q, h_kv = w.batch, w.s_q, w.h_q, w.h_kv
    hg = h_q // h_kv
    T = bt.shape[1] * 64
    j = torch.arange(T, device=q.device)
    srow = torch.arange(s_q, device=q.device).repeat_interleave(hg)                # row -> query token
    lim = sl.long()[:, None] - ((s_q - 1 - srow)[None, :] if w.causal else 0)      # [B, rows]
    valid = (j[None, None, :] < lim[:, :, None])[:, None]                          # [B, 1, rows, T]

    def run():
        kd = k[bt.long()].reshape(B, T, h_kv, 576).permute(0, 2, 1, 3)             # [B, h_kv, T, 576]
        qg = q.reshape(B, s_q, h_kv, hg, 576).permute(0, 2, 1, 3, 4).reshape(B, h_kv, s_q * hg, 576)
        s = torch.matmul(qg, kd.transpose(-1, -2)).float() * w.scale
        s = s.masked_fill(~valid, float("-inf"))
        lse = torch.logsumexp(s, dim=-1)
        p = torch.softmax(s, dim=-1).to(q.dtype)
        o = torch.matmul(p, kd[..., :512])
        return o, lse

    for _ in range(2):
        run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        run()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    return {"value": flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": ms, "reps": reps,
            "what": "PyTorch on this GPU: dense page gather, bf16 matmul Q.K^T, masked fp32 softmax and "
                    "logsumexp, bf16 matmul P.V (a comparison; the library never takes this path)"}


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    w = inputs.config(WORKLOADS[args.workload])
    per_step = []
    base = None
    budget = max(1.0, min(20.0, 120.0 / max(1, args.steps + args.warmup)))
    for i in range(args.warmup + args.steps):
        r = cpu_oracle_timing(w, budget_s=budget)
        if i >= args.warmup:
            per_step.append(r)
        base = r
    value = statistics.median(r["value"] for r in per_step)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * statistics.median(r["seconds"] for r in per_step),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, **w.describe()},
        "cpu_baseline": {k: base[k] for k in ("kind", "cores", "sample", "unit")} | {"value": value},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# The speed target of each large workload: its class and the fraction of the nominal B200 peak it is
# meant to reach, compute-bound configurations against 2.25 PFLOP/s dense bf16, the memory-bound one
# against 8 TB/s.
GATES = {
    "compute_bound": ("tensor", 0.5),
    "varlen_memory_bound": ("hbm", 0.7),
    "mtp_causal": ("tensor", 0.5),
    "long_context_split_kv": ("tensor", 0.5),
}
NOMINAL = {"tensor": (2250.0, "TFLOP/s"), "hbm": (8000.0, "GB/s")}
KERNEL_SAMPLES = 64          # back-to-back launches per kernel in the per-kernel loops
SIDE_STEPS = 200             # timed steps of each further workload in the default run


class Path:
    """One workload's device buffers and the three C-ABI launches of a decode step."""

    def __init__(self, w, dev, stream, lib):
        from mla_paged_kv_get_b200 import binding
        self.w, self.lib, self.stream = w, lib, stream
        self.q, self.k, self.bt, self.sl = (w.q.to(dev), w.k_cache.to(dev), w.block_table.to(dev),
                                            w.seqlens.to(dev))
        self.R, self.h_kv = w.rows_per_kv, w.h_kv
        self.G = binding.num_parts(self.R, self.h_kv)
        self.tile_md = torch.empty((self.G, 8), dtype=torch.int32, device=dev)
        self.num_splits = torch.empty((w.batch + 1,), dtype=torch.int32, device=dev)
        self.ws = torch.empty((binding.workspace_bytes(w.batch, self.R, self.h_kv, self.G),), dtype=torch.uint8,
                              device=dev)
        self.out = torch.empty((w.batch, w.s_q, w.h_q, 512), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((w.batch, w.s_q, w.h_q), dtype=torch.float32, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.h = binding._stream_handle(stream)
        self.P = binding._ptr
        self.binding = binding

    def metadata(self):
        w, P = self.w, self.P
        return self.lib.mla_get_metadata(P(self.sl), w.batch, self.R, self.h_kv, 0, P(self.tile_md),
                                         P(self.num_splits), None, self.h)

    def decode(self, flags=0):
        w, P = self.w, self.P
        return self.lib.mla_decode_paged_ex(
            P(self.q), P(self.k), self.k.shape[0], P(self.bt), self.bt.shape[1], P(self.sl), w.batch, w.s_q,
            w.h_q, self.h_kv, 576, 512, P(self.tile_md), P(self.num_splits), self.G, int(w.causal), w.scale,
            P(self.ws), self.ws.numel(), P(self.out), P(self.lse), P(self.status), flags, 0, self.h)

    def combine(self):
        w, P = self.w, self.P
        return self.lib.mla_combine(P(self.num_splits), P(self.ws), self.ws.numel(), w.batch, w.s_q, w.h_q,
                                    self.h_kv, self.G, P(self.out), P(self.lse), self.h)

    def step(self):
        """metadata + decode + combine: the public two-call API (mla_decode_paged launches the combine)."""
        return self.metadata() | self.decode(0)

    def check_status(self):
        st = int(self.status.item())
        assert st == 0, self.binding.status_string(st)

    def busy(self, seconds: float):
        """Untimed steps for about `seconds`, so the clocks sampled next are clocks under load."""
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < seconds:
            for _ in range(20):
                self.step()
            torch.cuda.synchronize()

    def kernel_ms(self, n: int = KERNEL_SAMPLES) -> dict:
        """Device time per launch of each kernel alone: n back-to-back launches of one kernel
        between two events on the launching stream (no event between launches, so each launch
        still overlaps its predecessor's tail through programmatic launch, as inside a step)."""
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        s = self.stream
        ev[0].record(s)
        for _ in range(n):
            self.metadata()
        ev[1].record(s)
        for _ in range(n):
            self.decode(2)     # decode kernel only; the partials stay in the workspace
        ev[2].record(s)
        for _ in range(n):
            self.combine()
        ev[3].record(s)
        torch.cuda.synchronize()
        self.step()            # leave complete results behind
        torch.cuda.synchronize()
        return {"metadata": ev[0].elapsed_time(ev[1]) / n, "decode": ev[1].elapsed_time(ev[2]) / n,
                "combine": ev[2].elapsed_time(ev[3]) / n, "samples": n}


def fractions(flops: int, nbytes: int, seconds: float, peaks) -> dict:
    tf = flops / seconds / 1e12
    gbs = nbytes / seconds / 1e9
    return {"tflops": tf, "hbm_gbs": gbs,
            "tensor_frac_of_2250": tf / 2250.0, "hbm_frac_of_8000": gbs / 8000.0,
            "tensor_frac_of_measured": tf / float(peaks["bf16_tflops"]),
            "hbm_frac_of_measured": gbs / float(peaks["hbm_gbs"])}


def gate(name: str, flops: int, nbytes: int, step_ms: float, decode_ms: float):
    """The speed target of this workload: its class, the target fraction and the fraction of the
    nominal peak reached by the whole step and by the decode kernel alone."""
    if name not in GATES:
        return {"class": "parity only (latency)", "step_us": step_ms * 1e3}
    cls, target = GATES[name]
    peak, unit = NOMINAL[cls]
    work = flops / 1e12 if cls == "tensor" else nbytes / 1e9
    f_step = work / (step_ms * 1e-3) / peak
    f_dec = work / (decode_ms * 1e-3) / peak
    return {"class": cls, "nominal_peak": peak, "unit": unit, "target_frac": target,
            "frac_step": f_step, "frac_decode_kernel": f_dec, "met": f_step >= target,
            "target_step_us": work / (target * peak) * 1e6}


def measure(path, steps: int, warmup: int, world: int, dev, peaks) -> dict:
    """Warm-up, then exactly `steps` timed steps between a barrier and a synchronize on both
    sides, the per-kernel loops and the clocks sampled over both."""
    w = path.w
    for _ in range(warmup):
        assert path.step() == 0
    torch.cuda.synchronize(dev)
    path.check_status()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev.index or 0)
    with sampler:
        path.busy(0.3)
        barrier(world)
        torch.cuda.synchronize(dev)
        start.record(path.stream)
        for _ in range(steps):
            path.step()
        stop.record(path.stream)
        torch.cuda.synchronize(dev)
        barrier(world)
        km = path.kernel_ms()
    path.check_status()
    ms_step = max_over_ranks(start.elapsed_time(stop) / steps, world, dev)
    decode_ms = max_over_ranks(km["decode"], world, dev)
    combine_ms = max_over_ranks(km["combine"], world, dev)
    metadata_ms = max_over_ranks(km["metadata"], world, dev)
    flops, nbytes = algorithmic_work(w)
    return {"w": w, "steps": steps, "ms_per_step": ms_step, "decode_ms": decode_ms, "combine_ms": combine_ms,
            "metadata_ms": metadata_ms, "kernel_samples": km["samples"], "flops": flops, "bytes": nbytes,
            "clocks": sampler.summary()}


def workload_entry(m: dict, peaks) -> dict:
    w = m["w"]
    return {
        "gate": gate(w.name, m["flops"], m["bytes"], m["ms_per_step"], m["decode_ms"]),
        "ms_per_step": m["ms_per_step"], "steps": m["steps"],
        "decode_us": m["decode_ms"] * 1e3, "combine_us": m["combine_ms"] * 1e3,
        "metadata_us": m["metadata_ms"] * 1e3, "kernel_samples": m["kernel_samples"],
        "algorithmic_flops": m["flops"], "algorithmic_bytes": m["bytes"],
        "step": fractions(m["flops"], m["bytes"], m["ms_per_step"] * 1e-3, peaks),
        "decode_kernel": fractions(m["flops"], m["bytes"], m["decode_ms"] * 1e-3, peaks),
        "launch_ms_le_step": m["decode_ms"] <= m["ms_per_step"],
        "config": {k: v for k, v in w.describe().items() if k != "workload"},
        "clocks": m["clocks"],
    }


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--workload", default=None, choices=sorted(WORKLOADS),
                    help="time this workload only (default: compute_bound as the headline, plus a "
                         "'workloads' entry for every other configuration)")
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-torch-baseline", action="store_true")
    args = ap.parse_args(argv)
    args.warmup = max(args.warmup, 3)
    only = args.workload is not None
    if args.workload is None:
        args.workload = DEFAULT_WORKLOAD

    world, rank, local = dist_setup()
    if args.impl == "reference":
        rc = run_reference(args, world, rank)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return rc

    from mla_paged_kv_get_b200 import binding
    lib = binding.load_library()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    peaks, peak_src = load_peaks()

    w = inputs.config(WORKLOADS[args.workload])
    path = Path(w, dev, stream, lib)
    m = measure(path, args.steps, args.warmup, world, dev, peaks)
    ms_step, decode_ms, flops, nbytes = m["ms_per_step"], m["decode_ms"], m["flops"], m["bytes"]
    # The decode kernel alone cannot take longer than the step that contains it.
    assert decode_ms <= ms_step * 1.02, (decode_ms, ms_step)

    # ---- end to end through the public API with host buffers (pinned), H2D + D2H inside the region
    hq, hk, hbt, hsl = (w.q.pin_memory(), w.k_cache.pin_memory(), w.block_table.pin_memory(),
                        w.seqlens.pin_memory())
    hout = torch.empty(path.out.shape, dtype=path.out.dtype).pin_memory()
    hlse = torch.empty(path.lse.shape, dtype=path.lse.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hbt, hsl))
    d2h = hout.numel() * hout.element_size() + hlse.numel() * hlse.element_size()
    e2e_steps = max(1, min(args.e2e_steps, args.steps))

    def e2e_step():
        path.q.copy_(hq, non_blocking=True)
        path.k.copy_(hk, non_blocking=True)
        path.bt.copy_(hbt, non_blocking=True)
        path.sl.copy_(hsl, non_blocking=True)
        assert path.step() == 0
        hout.copy_(path.out, non_blocking=True)
        hlse.copy_(path.lse, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize(dev)
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world, dev)
    path.check_status()

    hbm_peak = float(peaks["hbm_gbs"])
    tc_peak = float(peaks["bf16_tflops"])
    dec_s = decode_ms * 1e-3
    achieved_gbs = nbytes / dec_s / 1e9
    achieved_tf = flops / dec_s / 1e12
    t_hbm = nbytes / (hbm_peak * 1e9)
    t_tc = flops / (tc_peak * 1e12)
    bound = "hbm" if t_hbm >= t_tc else "tensor"
    traffic, traffic_sha = load_traffic(w.name)
    if traffic_sha is not None and traffic_sha != source_sha():
        traffic = None   # counters were taken on another version of the kernels
    roof = {"gate": gate(w.name, flops, nbytes, ms_step, decode_ms)}
    if bound == "hbm":
        roof.update({"bound": "hbm", "achieved": achieved_gbs, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved_gbs / hbm_peak})
    else:
        roof.update({"bound": "tensor", "achieved": achieved_tf, "peak": tc_peak, "unit": "TFLOP/s",
                     "frac": achieved_tf / tc_peak})
    roof.update({"traffic": traffic, "peak_source": f"{peak_src} (MEASURED_PEAKS.json burst)"
                 if peak_src == "measured" else "fallback",
                 "kernel": ("mla_decode_pair_kernel" if path.R > 64 else "mla_decode_kernel")
                 + f" ({m['kernel_samples']} back-to-back decode-only launches between CUDA events, after the "
                   "timed region)",
                 "launch_ms": decode_ms, "combine_ms": m["combine_ms"], "metadata_ms": m["metadata_ms"],
                 "launch_ms_le_step": decode_ms <= ms_step,
                 "algorithmic_bytes_per_launch": nbytes, "algorithmic_flops_per_launch": flops,
                 **{k: v for k, v in fractions(flops, nbytes, dec_s, peaks).items() if "frac" in k}})

    total_flops = flops * world
    line = {
        "metric": METRIC,
        "value": total_flops / (ms_step * 1e-3) / 1e12,
        "unit": "TFLOP/s",
        "hbm_gbs": nbytes * world / (ms_step * 1e-3) / 1e9,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {**w.describe(), "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": "inputs larger than L2: cache of %.0f MB per step vs 126 MB L2" % (nbytes / 1e6),
                   "step": "metadata + decode + combine"},
        "roofline": roof,
        "e2e": {"value": total_flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "ms_per_step": e2e_ms, "what": "pinned H2D of q, cache, page table, seqlens; "
                                             "metadata + decode + combine; D2H of out and lse"},
        "gpu_launches": 3 * args.steps,
        "clocks": m["clocks"],
    }
    del path
    if world == 1 and not only:
        # every other configuration, each in its own timed region of SIDE_STEPS steps
        side = {}
        for name in sorted(WORKLOADS, key=WORKLOADS.get):
            if name == w.name:
                continue
            wl = inputs.config(WORKLOADS[name])
            p = Path(wl, dev, stream, lib)
            side[name] = workload_entry(measure(p, SIDE_STEPS, args.warmup, world, dev, peaks), peaks)
            del p, wl
            torch.cuda.empty_cache()
        line["workloads"] = side
    if rank == 0 and world == 1 and not args.no_torch_baseline:
        line["torch_baseline"] = torch_native_timing(w, w.q.to(dev), w.k_cache.to(dev), w.block_table.to(dev),
                                                     w.seqlens.to(dev), flops)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_oracle_timing(w)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
