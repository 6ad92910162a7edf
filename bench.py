"""Benchmark of the vocab-sliced logits projection + per-row sampler on B200.

One step = one pass of the whole hot path over one batch: ``logits_local``
(tcgen05 GEMM, every vocab slice, no gather) followed by ``sample``
(temperature / top-k / top-p / Gumbel-max draw / top-n logprobs) on the
"decode" workload by default: 64 requests x 1 row, hidden 4096, vocab 151936
in 4 slices, bf16 hidden N(0,1) and lm_head N(0,0.02), per-request
T ~ U[0.5,1.5], top_k in {off,20,50}, top_p ~ U[0.8,1.0], top-20 logprobs.

Prints ONE JSON line (rank 0).  ``--impl reference`` times the CPU oracle on
the same workload instead.  Multi-GPU (torchrun): every rank runs its own
batch (weak scaling, no collective on the data path); the timed region is
bracketed by barriers and the max over ranks is reported.
"""
import argparse
import json
import os
import shutil
import signal
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from vocab_sharded_logits_b200 import workloads as W  # noqa: E402

L2_BYTES = 126 * 1024 * 1024


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# The timed units of a step and the sources each is built from.  "sample" is
# one call of the sampler: the streaming kernel (greedy and top-k <= 1024 rows)
# followed by the cluster kernel (the other rows).
_KERNEL_SOURCES = {"logits_local_kernel": ["vsl_gemm.cu"], "sample": ["vsl_sample.cu", "vsl_stream.cuh"]}


def _source_sha(kernel):
    import hashlib
    h = hashlib.sha256()
    for name in _KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "vocab_sharded_logits_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def _recorded_traffic(kernel, workload):
    """DRAM bytes per call recorded from an ncu capture in profiles/<kernel>_<workload>.md,
    or None when there is none or the sources changed since (sha256 over them differs)."""
    prof = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    if not os.path.exists(prof):
        return None
    fields = {}
    for line in open(prof):
        if ":" in line and line.split(":", 1)[0] in ("traffic_bytes_per_launch", "source_sha256"):
            k, v = line.split(":", 1)
            fields[k] = v.strip()
    if fields.get("source_sha256") != _source_sha(kernel):
        return None
    try:
        return int(fields["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """Samples nvidia-smi SM clocks and throttle reasons during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.idx = device_index
        self.proc = None
        self.path = None
        self.skip = 0

    def start(self):
        """Starts sampling and waits (up to 5 s) until the first sample is written."""
        if shutil.which("nvidia-smi") is None:
            return
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                                      "-i", str(self.idx), "-lms", "50"], stdout=open(self.path, "w"),
                                     stderr=subprocess.DEVNULL)
        t0 = time.time()
        while time.time() - t0 < 5 and os.path.getsize(self.path) == 0:
            time.sleep(0.02)
        self.skip = self.count()

    def count(self):
        if self.path is None:
            return 0
        with open(self.path) as f:
            return sum(1 for _ in f)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.send_signal(signal.SIGTERM)
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        lines = open(self.path).read().splitlines()[self.skip:]   # samples taken while the steps ran
        for line in lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons), "samples": len(sm)}


def _dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def _max_over_ranks(x, world, device):
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def cpu_oracle_rows(w, n_rows, seed=0):
    """Times the oracle on ``n_rows`` rows of workload ``w`` (projection + sampler).

    Returns (seconds, rows, threads).  Inputs are made on the CPU from the same
    seeded recipe; only the oracle calls are timed.
    """
    from oracle.gemm import logits_local as ref_logits
    from oracle.sampler import sample_row
    hidden, ws = W.gemm_inputs(W.scaled(w, requests=max(1, n_rows // w.rows_per_request)), "cpu")
    h = hidden.float().numpy()[:n_rows]
    ws_np = [x.float().numpy() for x in ws]
    T, k, p, req, pos = W.row_params(w)
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        threads = os.cpu_count() or 1
    t0 = time.perf_counter()
    logits = np.concatenate(ref_logits(h, ws_np), axis=1).astype(np.float32)
    for r in range(n_rows):
        sample_row(logits[r], T[r], int(k[r]), p[r], int(req[r]), int(pos[r]), seed, w.n_logprobs)
    return time.perf_counter() - t0, n_rows, threads


def run_reference(args, w):
    world, rank, _ = _dist_setup(args.gpus)
    if rank != 0:
        return 0
    for _ in range(args.warmup):
        cpu_oracle_rows(w, 1)
    times, rows = [], 0
    for _ in range(args.steps):
        t, n, threads = cpu_oracle_rows(w, args.reference_rows)
        times.append(t)
        rows += n
    total = sum(times)
    value = rows / total
    line = {
        "impl": "reference", "metric": _metric(w), "value": value, "unit": "rows/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": _config(w),
        "cpu_baseline": {"value": value, "unit": "rows/s", "cores": threads, "kind": "oracle",
                         "sample": f"{args.reference_rows} rows per step of the {w.name} workload "
                                   f"(float64 projection of those rows over all {w.V} tokens + the sampler oracle)"},
        "e2e": {"value": value, "unit": "rows/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def _e2e_sizes(R, H, n):
    """Bytes of the packed per-step input (bf16 hidden [R, H], then int32 row
    parameters [R, 5]) and int32 words of the packed output (token ids, token
    logprobs, top-n ids, top-n logprobs, row flags) of the end-to-end leg."""
    return R * H * 2 + R * 5 * 4, R * (3 + 2 * n)


def _e2e_views(buf_in, buf_out, R, H, n):
    """hidden, params and a SampleResult viewing one packed input buffer (uint8)
    and one packed output buffer (int32), so each step moves one block each way."""
    import vocab_sharded_logits_b200 as vsl
    hid = buf_in[: R * H * 2].view(torch.bfloat16).view(R, H)
    prm = buf_in[R * H * 2:].view(torch.int32).view(R, 5)
    res = vsl.SampleResult(buf_out[:R], buf_out[R:2 * R].view(torch.float32),
                           buf_out[2 * R:2 * R + R * n].view(R, n),
                           buf_out[2 * R + R * n:2 * R + 2 * R * n].view(torch.float32).view(R, n),
                           buf_out[2 * R + 2 * R * n:])
    return hid, prm, res


def _metric(w):
    return f"sampled rows/sec ({w.name}: logits_local GEMM + sampler, V={w.V})"


def _config(w):
    return {"workload": w.name, "requests": w.requests, "rows": w.R, "hidden": w.H, "vocab": w.V, "slices": w.S,
            "n_logprobs": w.n_logprobs, "l2": "inputs larger than L2 (lm_head weights "
            f"{w.V * w.H * 2 / 1e9:.3f} GB read per step); sampler-only figure flushes L2 between reps"}


def run_gpu(args, w):
    import vocab_sharded_logits_b200 as vsl
    world, rank, local = _dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    hbm_peak, tf_peak, tf_sus, peak_kind = _peaks()

    hidden, ws = W.gemm_inputs(w, dev)
    T, k, p, req, pos = W.row_params(w)
    params = vsl.make_row_params(T, k, p, req + rank * w.requests, pos, dev)
    logits = [torch.empty(w.R, w.V_s, dtype=torch.float32, device=dev) for _ in range(w.S)]
    n = w.n_logprobs
    out = vsl.SampleResult(torch.empty(w.R, dtype=torch.int32, device=dev), torch.empty(w.R, device=dev),
                           torch.empty(w.R, n, dtype=torch.int32, device=dev), torch.empty(w.R, n, device=dev),
                           torch.empty(w.R, dtype=torch.int32, device=dev))

    def step(seed):
        vsl.logits_local(hidden, ws, out=logits, stream=stream)
        vsl.sample(logits, params, seed, n, out=out, stream=stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()

    # ---- timed region: K steps, per-kernel events on the launching stream
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    clocks = ClockSampler(local)
    clocks.start()
    _barrier(world)
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        a, b, c = ev[i]
        a.record(stream)
        vsl.logits_local(hidden, ws, out=logits, stream=stream)
        b.record(stream)
        vsl.sample(logits, params, 1000 + i, n, out=out, stream=stream)
        c.record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    # a timed region shorter than the sampling period still gets samples: keep
    # running the same step (untimed) until three samples under load exist
    t0 = time.time()
    while clocks.proc is not None and clocks.count() - clocks.skip < 3 and time.time() - t0 < 10:
        for i in range(20):
            step(5000 + i)
        torch.cuda.synchronize()
    _barrier(world)
    clk = clocks.stop()
    total_ms = t_start.elapsed_time(t_end)
    gemm_ms = sum(a.elapsed_time(b) for a, b, _ in ev) / args.steps
    samp_ms = sum(b.elapsed_time(c) for _, b, c in ev) / args.steps
    total_ms = _max_over_ranks(total_ms, world, dev)
    ms_per_step = total_ms / args.steps
    value = world * w.R * args.steps / (total_ms / 1e3)

    # ---- sampler alone with L2 flushed between reps (its HBM figure)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    s_times = []
    for i in range(max(3, args.steps)):
        flush.fill_(float(i))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        vsl.sample(logits, params, 2000 + i, n, out=out, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize()
        s_times.append(e0.elapsed_time(e1))
    samp_cold_ms = statistics.median(s_times)
    del flush

    # ---- end to end through the public API with host buffers.  Every step copies
    # its inputs (hidden states + row parameters, one packed pinned buffer) to the
    # device and reads its results (one packed buffer of the five outputs) back.
    # The copies run on a copy stream, double-buffered, so step i + 1's inputs
    # cross PCIe while step i computes: the way a serving loop feeds the GPU.
    in_bytes, out_words = _e2e_sizes(w.R, w.H, n)
    h2d, d2h = in_bytes, out_words * 4
    pin_in = [torch.empty(in_bytes, dtype=torch.uint8).pin_memory() for _ in range(2)]
    for b in range(2):
        pin_in[b][: w.R * w.H * 2].view(torch.bfloat16).view(w.R, w.H).copy_(hidden.cpu())
        pin_in[b][w.R * w.H * 2:].view(torch.int32).view(w.R, 5).copy_(params.cpu())
    pin_out = [torch.empty(out_words, dtype=torch.int32).pin_memory() for _ in range(2)]
    dev_in = [torch.empty(in_bytes, dtype=torch.uint8, device=dev) for _ in range(2)]
    dev_out = [torch.empty(out_words, dtype=torch.int32, device=dev) for _ in range(2)]

    bufs = [_e2e_views(dev_in[b], dev_out[b], w.R, w.H, n) for b in range(2)]
    copy_stream = torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]    # inputs of buffer b are on the device
    ev_done = [torch.cuda.Event() for _ in range(2)]  # the step using buffer b has computed
    ev_out = [torch.cuda.Event() for _ in range(2)]   # results of buffer b are on the host

    def e2e_run(first_seed, steps, start=None):
        if start is not None:
            copy_stream.wait_event(start)  # no copy of the timed steps starts before the clock
        for b in range(2):
            ev_out[b].record(copy_stream)
        for i in range(steps):
            b = i & 1
            hid, prm, res = bufs[b]
            with torch.cuda.stream(copy_stream):
                copy_stream.wait_event(ev_out[b])  # buffer b's previous step has been read back
                dev_in[b].copy_(pin_in[b], non_blocking=True)
                ev_in[b].record(copy_stream)
            stream.wait_event(ev_in[b])
            vsl.logits_local(hid, ws, out=logits, stream=stream)
            vsl.sample(logits, prm, first_seed + i, n, out=res, stream=stream)
            ev_done[b].record(stream)
            with torch.cuda.stream(copy_stream):
                copy_stream.wait_event(ev_done[b])
                pin_out[b].copy_(dev_out[b], non_blocking=True)
                ev_out[b].record(copy_stream)
        for b in range(2):
            stream.wait_event(ev_out[b])  # every result is on the host

    e2e_run(0, args.warmup)
    torch.cuda.synchronize()
    _barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_run(3000, args.steps, e0)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = _max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e_value = world * w.R * args.steps / (e2e_ms / 1e3)
    _barrier(world)

    status = vsl.device_error()
    if status != (0, 0):
        print(f"device error word set: {status}", file=sys.stderr)

    # ---- roofline of the dominant kernel
    gemm_bytes = w.V * w.H * 2 + w.R * w.H * 2 + w.R * w.V * 4
    gemm_flops = 2.0 * w.R * w.H * w.V
    samp_bytes = w.R * w.V * 4
    intensity = gemm_flops / gemm_bytes
    ridge = tf_peak * 1e12 / (hbm_peak * 1e9)
    if gemm_ms >= samp_ms:
        if intensity < ridge:
            roof = {"kernel": "logits_local_kernel", "bound": "hbm", "achieved": gemm_bytes / (gemm_ms / 1e3) / 1e9,
                    "peak": hbm_peak, "unit": "GB/s"}
        else:
            roof = {"kernel": "logits_local_kernel", "bound": "tensor", "achieved": gemm_flops / (gemm_ms / 1e3) / 1e12,
                    "peak": tf_sus, "unit": "TFLOP/s"}
    else:
        roof = {"kernel": "sample", "bound": "hbm", "achieved": samp_bytes / (samp_ms / 1e3) / 1e9,
                "peak": hbm_peak, "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["peak_source"] = peak_kind
    roof["traffic"] = _recorded_traffic(roof["kernel"], w.name)

    line = {
        "metric": _metric(w), "value": value, "unit": "rows/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": _config(w),
        "roofline": roof,
        "kernels": {
            "logits_local_ms": gemm_ms, "sample_ms": samp_ms, "sample_cold_l2_ms": samp_cold_ms,
            "gemm_tflops": gemm_flops / (gemm_ms / 1e3) / 1e12,
            "gemm_hbm_gbs": gemm_bytes / (gemm_ms / 1e3) / 1e9,
            "sampler_rows_per_s": w.R / (samp_ms / 1e3),
            "sampler_hbm_gbs_cold_l2": samp_bytes / (samp_cold_ms / 1e3) / 1e9,
            "sampler_hbm_gbs_in_step": samp_bytes / (samp_ms / 1e3) / 1e9,
        },
        "e2e": {"value": e2e_value, "unit": "rows/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": (1 + vsl.sample_launches(w.R, w.S, w.V_s)) * args.steps,  # projection + sampler kernels
        "clocks": clk,
        "cpu_baseline": None,
    }
    if rank == 0 and world == 1 and not args.skip_cpu:
        secs, rows, threads = cpu_oracle_rows(w, args.cpu_rows)
        line["cpu_baseline"] = {"value": rows / secs, "unit": "rows/s", "cores": threads, "kind": "oracle",
                                "sample": f"{rows} rows of the {w.name} workload: float64 projection of those rows "
                                          f"over all {w.V} tokens + the sampler oracle ({secs:.1f} s)"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def run_sampler_only(args, w):
    """Times ``sample`` alone on the workload's synthetic fp32 logits (the recipe of
    the parity tests), L2 flushed before every rep; prints one JSON line."""
    import vocab_sharded_logits_b200 as vsl
    dev = torch.device("cuda", 0)
    hbm_peak, _, _, peak_kind = _peaks()
    logits = W.sampler_logits(w, dev)
    slices = [t.contiguous() for t in torch.tensor_split(logits, w.S, dim=1)]
    del logits
    T, k, p, req, pos = W.row_params(w)
    params = vsl.make_row_params(T, k, p, req, pos, dev)
    out = vsl.sample(slices, params, 0, w.n_logprobs)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    for i in range(args.warmup):
        vsl.sample(slices, params, i, w.n_logprobs, out=out)
    times = []
    for i in range(args.steps):
        flush.fill_(float(i))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        vsl.sample(slices, params, 100 + i, w.n_logprobs, out=out)
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    ms = statistics.median(times)
    nbytes = w.R * w.V * 4
    print(json.dumps({"metric": f"sampler rows/sec ({w.name}, V={w.V}, L2 flushed)", "value": w.R / (ms / 1e3),
                      "unit": "rows/s", "ms": ms, "hbm_gbs": nbytes / (ms / 1e3) / 1e9,
                      "roofline": {"bound": "hbm", "achieved": nbytes / (ms / 1e3) / 1e9, "peak": hbm_peak,
                                   "unit": "GB/s", "frac": nbytes / (ms / 1e3) / 1e9 / hbm_peak,
                                   "peak_source": peak_kind},
                      "config": {"workload": w.name, "rows": w.R, "vocab": w.V, "slices": w.S}}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["vsl", "reference"], default="vsl")
    ap.add_argument("--workload", default="decode", choices=sorted(W.WORKLOADS))
    ap.add_argument("--cpu-rows", type=int, default=4)
    ap.add_argument("--reference-rows", type=int, default=2)
    ap.add_argument("--skip-cpu", action="store_true")
    ap.add_argument("--sampler-only", action="store_true",
                    help="time the sampler alone on the workload's synthetic logits (profiling aid)")
    args = ap.parse_args()
    w = W.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    if not torch.cuda.is_available():
        print(json.dumps({"error": "no CUDA device"}))
        return 1
    if args.sampler_only:
        return run_sampler_only(args, w)
    return run_gpu(args, w)


if __name__ == "__main__":
    sys.exit(main())
