"""Throughput of one MLA paged-decode step on B200, as one JSON line.

A step is the whole hot path over one batch: the metadata kernel, the split-KV
decode kernel and the combine kernel, launched through the C ABI on one
stream.  The default workload is the compute-bound decode configuration
(64 sequences x 4096 tokens, h_q = 128, one shared 576-wide KV head, 64-token
pages, shuffled page table); its 302 MB cache is larger than the 126 MB L2,
so consecutive steps do not hit in L2.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl reference]

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


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-torch-baseline", action="store_true")
    args = ap.parse_args(argv)
    args.warmup = max(args.warmup, 3)

    world, rank, local = dist_setup()
    if args.impl == "reference":
        rc = run_reference(args, world, rank)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return rc

    from mla_paged_kv_get_b200 import binding
    binding.load_library()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)

    idx = WORKLOADS[args.workload]
    w = inputs.config(idx)
    flops, nbytes = algorithmic_work(w)
    q, k, bt, sl = (w.q.to(dev), w.k_cache.to(dev), w.block_table.to(dev), w.seqlens.to(dev))
    R, h_kv = w.rows_per_kv, w.h_kv
    G = binding.num_parts(R, h_kv)
    tile_md = torch.empty((G, 8), dtype=torch.int32, device=dev)
    num_splits = torch.empty((w.batch + 1,), dtype=torch.int32, device=dev)
    ws = torch.empty((binding.workspace_bytes(w.batch, R, h_kv, G),), dtype=torch.uint8, device=dev)
    out = torch.empty((w.batch, w.s_q, w.h_q, 512), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.batch, w.s_q, w.h_q), dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    lib = binding.load_library()
    h = binding._stream_handle(stream)
    P = binding._ptr

    def step():
        rc = lib.mla_get_metadata(P(sl), w.batch, R, h_kv, 0, P(tile_md), P(num_splits), None, h)
        rc |= lib.mla_decode_paged(P(q), P(k), k.shape[0], P(bt), bt.shape[1], P(sl), w.batch, w.s_q, w.h_q,
                                   h_kv, 576, 512, P(tile_md), P(num_splits), G, int(w.causal),
                                   w.scale, P(ws), ws.numel(), P(out), P(lse), P(status), h)
        return rc

    # events between the launches give per-kernel device time inside the timed region
    def step_with_events(ev):
        lib.mla_get_metadata(P(sl), w.batch, R, h_kv, 0, P(tile_md), P(num_splits), None, h)
        ev[0].record(stream)
        lib.mla_decode_paged_ex(P(q), P(k), k.shape[0], P(bt), bt.shape[1], P(sl), w.batch, w.s_q, w.h_q,
                                h_kv, 576, 512, P(tile_md), P(num_splits), G, int(w.causal),
                                w.scale, P(ws), ws.numel(), P(out), P(lse), P(status), 2, 0, h)
        ev[1].record(stream)
        lib.mla_combine(P(num_splits), P(ws), ws.numel(), w.batch, w.s_q, w.h_q, h_kv, G, P(out), P(lse), h)
        ev[2].record(stream)

    for _ in range(args.warmup):
        assert step() == 0
    torch.cuda.synchronize(dev)
    assert int(status.item()) == 0, binding.status_string(int(status.item()))

    # ---- timed region: K steps, barrier + sync on both sides.  Every EV_EVERY-th step carries
    # events around the decode and combine launches (on the launching stream).  An event between
    # two launches breaks their programmatic-launch overlap, so the instrumented steps are slower
    # than the rest: they are kept few (500 steps -> 32 samples of each kernel).
    EV_EVERY = 16
    n_ev = min((args.steps + EV_EVERY - 1) // EV_EVERY, 512)
    evs = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(n_ev)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize(dev)
    with sampler:
        start.record(stream)
        for i in range(args.steps):
            if i % EV_EVERY == 0 and i // EV_EVERY < n_ev:
                step_with_events(evs[i // EV_EVERY])
            else:
                step()
        stop.record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    ms_total = start.elapsed_time(stop)
    ms_total_max = max_over_ranks(ms_total, world, dev)
    ms_step = ms_total_max / args.steps
    decode_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)    # decode kernel alone
    combine_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    assert int(status.item()) == 0, binding.status_string(int(status.item()))

    # ---- end to end through the public API with host buffers (pinned), H2D + D2H inside the region
    hq, hk, hbt, hsl = (w.q.pin_memory(), w.k_cache.pin_memory(), w.block_table.pin_memory(),
                        w.seqlens.pin_memory())
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    hlse = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hbt, hsl))
    d2h = hout.numel() * hout.element_size() + hlse.numel() * hlse.element_size()
    e2e_steps = max(1, min(args.e2e_steps, args.steps))

    def e2e_step():
        q.copy_(hq, non_blocking=True)
        k.copy_(hk, non_blocking=True)
        bt.copy_(hbt, non_blocking=True)
        sl.copy_(hsl, non_blocking=True)
        assert step() == 0
        hout.copy_(out, non_blocking=True)
        hlse.copy_(lse, non_blocking=True)

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

    peaks, peak_src = load_peaks()
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
    if bound == "hbm":
        roof = {"bound": "hbm", "achieved": achieved_gbs, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved_gbs / hbm_peak}
    else:
        roof = {"bound": "tensor", "achieved": achieved_tf, "peak": tc_peak, "unit": "TFLOP/s",
                "frac": achieved_tf / tc_peak}
    roof.update({"traffic": traffic, "peak_source": f"{peak_src} (MEASURED_PEAKS.json burst)"
                 if peak_src == "measured" else "fallback",
                 "kernel": ("mla_decode_pair_kernel" if R > 64 else "mla_decode_kernel")
                 + f" (CUDA events around its launch on every {EV_EVERY}th timed step)",
                 "combine_ms": combine_ms,
                 "algorithmic_bytes_per_launch": nbytes, "algorithmic_flops_per_launch": flops,
                 "launch_ms": decode_ms,
                 "tensor_frac_of_measured": achieved_tf / tc_peak,
                 "hbm_frac_of_measured": achieved_gbs / hbm_peak,
                 "tensor_frac_of_2250": achieved_tf / 2250.0, "hbm_frac_of_8000": achieved_gbs / 8000.0})

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
        "clocks": sampler.summary(),
    }
    if rank == 0 and world == 1 and not args.no_torch_baseline:
        line["torch_baseline"] = torch_native_timing(w, q, k, bt, sl, flops)
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
