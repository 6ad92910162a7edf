"""Benchmark of the vocab-sliced logits projection + per-row sampler on B200.

One step = one pass of the whole hot path over one batch: ``logits_local``
(tcgen05 GEMM, every vocab slice, no gather) followed by ``sample``
(temperature / top-k / top-p / Gumbel-max draw / top-n logprobs).  The
headline line is the "large batch" workload by default: 256 requests x 8 rows
(7 speculative tokens + 1) = 2048 rows, hidden 5120, vocab 151936 in 8 slices,
bf16 hidden N(0,1) and lm_head N(0,0.02), per-request T ~ U[0.3,1.2],
top_p ~ U[0.5,1.0], top_k off, top-20 logprobs.  The same line carries
``per_config``: every workload measured in the same run (projection TFLOP/s,
sampler GB/s with L2 flushed, rows/s in the step and end to end).

Prints ONE JSON line (rank 0).  ``--impl reference`` times the CPU sampler
oracle on the same workload instead.  Multi-GPU (torchrun): every rank runs its
own batch (weak scaling, no collective on the data path); every timed region
is bracketed by barriers and the max over ranks is reported.
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

import workloads as W  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
METRIC = "sampled rows/sec and sampler HBM GB/s at V=151936; logits-GEMM TFLOPS on 1 B200"
# every workload measured into per_config, in this order (the headline's first)
PER_CONFIG = ["tiny", "decode", "spec", "large", "peaked", "wide"]
PARITY_SEED = 777


def _peaks():
    """(HBM GB/s, bf16 TF/s burst, bf16 TF/s sustained, source)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# The timed units of a step and the sources each is built from.  "sample" is
# one call of the sampler (the streaming kernel and the cluster kernel).
_KERNEL_SOURCES = {"logits_local_kernel": ["vsl_gemm.cu", "vsl_ptx.cuh"],
                   "sample": ["vsl_sample.cu", "vsl_stream.cuh", "vsl_math.cuh", "vsl_ptx.cuh"]}


def _source_sha(kernel):
    import hashlib
    h = hashlib.sha256()
    for name in _KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "vocab_sharded_logits_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def _recorded_traffic(kernel, workload, profiles_dir=None):
    """DRAM bytes per call recorded from an ncu capture in profiles/<kernel>_<workload>.md,
    or None when there is none or the sources changed since (sha256 over them differs)."""
    prof = os.path.join(profiles_dir or os.path.join(ROOT, "profiles"), f"{kernel}_{workload}.md")
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


# ------------------------------------------------------------------ the CPU oracle

def _nproc():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_baseline(logits_np, params, seed, n_logprobs, label, gpu_tokens=None, budget_s=2.0, reps=5):
    """The sampler oracle, as it stands, timed on this host's cores over rows of
    ``logits_np`` (float32 [rows, V]): one thread, then one worker per core (rows
    split between them), wall clock, median of ``reps`` runs of about ``budget_s``
    each.  Returns the ``cpu_baseline`` object and, when ``gpu_tokens`` is given,
    a token parity summary of the GPU's draw (same logits, same seed) against the
    oracle's on every row the all-cores runs sampled."""
    from oracle.timing import OracleSampler, cpu_model
    rows_avail = logits_np.shape[0]
    nproc = _nproc()
    orc = OracleSampler(logits_np, params, seed, n_logprobs, workers=nproc)
    try:
        t, _ = orc.run([0], parallel=False)          # warm-up and a first estimate
        t, _ = orc.run([min(1, rows_avail - 1)], parallel=False)
        per_row = max(t, 1e-4)
        n1 = max(2, min(rows_avail, int(budget_s / per_row)))
        rate1, med1, _ = orc.median_rate(range(n1), parallel=False, reps=reps)
        orc.start_workers()
        n_all = max(nproc, min(4 * rows_avail, nproc * max(1, int(budget_s / per_row))))
        rows_all = [r % rows_avail for r in range(n_all)]
        rate_all, med_all, res = orc.median_rate(rows_all, parallel=True, reps=reps)
    finally:
        orc.close()
    base = {"value": rate_all, "unit": "rows/s", "cores": nproc, "kind": "oracle",
            "sample": f"{label}: the sampler oracle (float64, sort based) over rows of the same fp32 logits; "
                      f"all cores: {n_all} rows per run on {nproc} worker processes ({med_all:.2f} s); one thread: "
                      f"{n1} rows per run ({med1:.2f} s); median of {reps} runs each",
            "threads_1": rate1, "threads_all": rate_all, "nproc": nproc, "cpu_model": cpu_model()}
    parity = None
    if gpu_tokens is not None:
        seen = {}
        for r, tok, near, cut, flags in res:
            seen[r] = (tok, near, cut, flags)
        eq = sum(1 for r, (tok, _, _, _) in seen.items() if int(gpu_tokens[r]) == tok)
        near = sum(1 for v in seen.values() if v[1])
        cut = sum(1 for v in seen.values() if v[2])
        unexplained = sum(1 for r, (tok, nt, ct, _) in seen.items() if int(gpu_tokens[r]) != tok and not (nt or ct))
        parity = {"rows": len(seen), "token_equal": eq, "near_tie": near, "cut_tie": cut,
                  "mismatch_unexplained": unexplained, "seed": seed}
    return base, parity


def run_reference(args, w):
    """The oracle arm: the sampler oracle on the host's cores, each step a bounded
    sample of the workload's rows (synthetic fp32 logits with the spread of the
    projection's output), all cores."""
    world, rank, _ = _dist_setup(args.gpus)
    if rank != 0:
        return 0
    from oracle.timing import OracleSampler, cpu_model
    nproc = _nproc()
    rows = max(1, min(w.R, args.reference_rows * nproc))
    wl = W.scaled(w, requests=max(1, -(-rows // w.rows_per_request)))
    logits = W.sampler_logits(wl, "cpu").numpy()[:rows]
    params = W.row_params(w)
    orc = OracleSampler(logits, params, 0, w.n_logprobs, workers=nproc)
    try:
        orc.start_workers()
        for _ in range(args.warmup):
            orc.run(range(min(rows, nproc)), parallel=True)
        times = []
        for _ in range(args.steps):
            t, _ = orc.run(range(rows), parallel=True)
            times.append(t)
    finally:
        orc.close()
    total = sum(times)
    value = rows * args.steps / total
    sample = (f"{rows} rows per step of the {w.name} workload (V={w.V}): the sampler oracle over synthetic fp32 "
              f"logits with the projection's spread, {nproc} worker processes")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "rows/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": _config(w),
        "cpu_baseline": {"value": value, "unit": "rows/s", "cores": nproc, "kind": "oracle", "sample": sample,
                         "nproc": nproc, "cpu_model": cpu_model()},
        "e2e": {"value": value, "unit": "rows/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ the GPU arm

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


def _config(w):
    return {"workload": w.name, "requests": w.requests, "rows": w.R, "hidden": w.H, "vocab": w.V, "slices": w.S,
            "n_logprobs": w.n_logprobs,
            "sampler_input": "synthetic peaked / long-tail logits" if w.name == "peaked" else "the projection's output",
            "l2": "inputs larger than L2 in the step (lm_head weights "
                  f"{w.V * w.H * 2 / 1e9:.3f} GB read per step); the sampler-alone figures flush L2 (a 252 MB "
                  "write) before every rep"}


def _events(n):
    return [torch.cuda.Event(enable_timing=True) for _ in range(n)]


def _tile_rows(T, k, V):
    """Rows the sampler's tile mode takes: greedy, or 0 < top_k <= 1024 (below V)."""
    T = np.asarray(T, np.float32)
    k = np.asarray(k, np.int64)
    return (T == 0) | ((k > 0) & (k < V) & (k <= 1024))


def _large_batch(w, sms):
    """More rows than SMs: the streaming kernel gives each row one CTA and also
    takes the top-k-off rows (which then read the records too)."""
    return w.R > sms


def _uses_tiles(w, T, k, sms):
    """The step requests tile statistics when some row can use them (and the
    vocabulary has at most 4096 blocks of 128)."""
    some = bool(_tile_rows(T, k, w.V).any()) or _large_batch(w, sms)
    return some and w.S * (-(-w.V_s // 128)) <= 4096


def _sampler_read_bytes(w, T, k, stats, sms):
    """Algorithmic bytes one sampler call reads.  Without records every row
    reads its V logits.  With them, a greedy or top-k row reads its records
    (S * B * 32 bytes) and the 32-logit quarters whose largest x reaches
    fl(t0 / T), t0 the R-th largest block maximum, R = max(n, k) (greedy:
    max(n, 1)); a top-k-off row of a large batch its records and its V logits
    once (the top-p passes; its few top-n quarters are not counted); any other
    row its V logits.  The quarters are counted from the records with torch on
    the device (the kernel's cut can sit a few floats lower, where the
    temperature maps neighbours to one x: an undercount of a few quarters at
    most)."""
    tile = _tile_rows(T, k, w.V)
    if stats is None:
        return w.R * w.V * 4
    SB = w.S * (-(-w.V_s // 128))
    koff = int((~tile).sum())
    full = koff * (w.V * 4 + (SB * 32 if _large_batch(w, sms) else 0))
    if not tile.any():
        return full
    dev = stats.device
    rows = torch.from_numpy(np.flatnonzero(tile)).to(dev)
    st = stats[rows]
    SB = st.shape[1]
    Tt = torch.as_tensor(np.asarray(T, np.float32)[tile], device=dev)
    kt = torch.as_tensor(np.asarray(k, np.int64)[tile], device=dev)
    n = max(w.n_logprobs, 1)
    r_sel = torch.where(Tt == 0, torch.full_like(kt, n), torch.clamp(kt, min=w.n_logprobs))
    qmax = st[..., :4]
    bmax = qmax.amax(-1).sort(dim=1, descending=True).values
    t0 = bmax.gather(1, (r_sel - 1).clamp(max=SB - 1)[:, None]).squeeze(1)
    t0 = torch.where(r_sel > SB, torch.full_like(t0, -float("inf")), t0)
    scale = torch.where(Tt == 0, torch.ones_like(Tt), Tt)
    sel = (qmax / scale[:, None, None]) >= (t0 / scale)[:, None, None]
    quarters = int(sel.sum())
    return full + int(tile.sum()) * SB * 32 + quarters * 128


def measure_config(w, dev, world, rank, steps, warmup, peaks):
    """One workload on this rank: the timed steps (projection + sampler, events per
    kernel on the launching stream), the sampler alone with L2 flushed, the end-to-end
    leg through the public API with host buffers.  Times are maxima over ranks.
    Returns (summary dict, state for the headline's extra legs)."""
    import vocab_sharded_logits_b200 as vsl
    hbm_peak, tf_peak, _, _ = peaks
    stream = torch.cuda.current_stream(dev)
    hidden, ws = W.gemm_inputs(w, dev)
    T, k, p, req, pos = W.row_params(w)
    params = vsl.make_row_params(T, k, p, req + rank * w.requests, pos, dev)
    logits = [torch.empty(w.R, w.V_s, dtype=torch.float32, device=dev) for _ in range(w.S)]
    # the peaked workload's sampler reads its own synthetic logits; the others sample the projection's output
    samp_in = logits
    if w.name == "peaked":
        samp_in = [t.contiguous() for t in torch.tensor_split(W.sampler_logits(w, dev), w.S, dim=1)]
    n = w.n_logprobs
    out = vsl.SampleResult(torch.empty(w.R, dtype=torch.int32, device=dev), torch.empty(w.R, device=dev),
                           torch.empty(w.R, n, dtype=torch.int32, device=dev), torch.empty(w.R, n, device=dev),
                           torch.empty(w.R, dtype=torch.int32, device=dev))
    # tile statistics, when some row can use them: the projection writes them
    # every step and the sampler reads them; for the peaked workload, whose
    # sampler reads its own synthetic logits, the records of those logits
    # (written once) stand in for the epilogue's
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    tiles = _uses_tiles(w, T, k, sms)
    stats = torch.empty(vsl.tile_stats_shape(w.R, w.S, w.V_s), device=dev) if tiles else None
    samp_stats = vsl.tile_stats(samp_in) if tiles and samp_in is not logits else stats

    def project(hid, stream):
        vsl.logits_local(hid, ws, out=logits, stream=stream, tile_stats=stats)

    def sample(prm, seed, res, stream):
        vsl.sample(samp_in, prm, seed, n, out=res, stream=stream, tile_stats=samp_stats)

    def step(seed):
        project(hidden, stream)
        sample(params, seed, out, stream)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    ev = [_events(3) for _ in range(steps)]
    _barrier(world)
    torch.cuda.synchronize()
    t0, t1 = _events(2)
    t0.record(stream)
    for i in range(steps):
        a, b, c = ev[i]
        a.record(stream)
        project(hidden, stream)
        b.record(stream)
        sample(params, 1000 + i, out, stream)
        c.record(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    total_ms = _max_over_ranks(t0.elapsed_time(t1), world, dev)
    gemm_ms = _max_over_ranks(sum(a.elapsed_time(b) for a, b, _ in ev) / steps, world, dev)
    samp_ms = _max_over_ranks(sum(b.elapsed_time(c) for _, b, c in ev) / steps, world, dev)

    # the sampler alone, L2 flushed before every rep (its HBM figure)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    s_times = []
    for i in range(max(5, steps)):
        flush.fill_(float(i))
        e0, e1 = _events(2)
        e0.record(stream)
        sample(params, 2000 + i, out, stream)
        e1.record(stream)
        torch.cuda.synchronize()
        s_times.append(e0.elapsed_time(e1))
    del flush
    samp_cold_ms = _max_over_ranks(statistics.median(s_times), world, dev)

    # end to end through the public API with host buffers: every step copies its
    # inputs (hidden states + row parameters, one packed pinned buffer) to the
    # device and reads its results (one packed buffer of the five outputs) back,
    # double-buffered, the uploads and the read-backs on two copy streams of
    # their own (on one stream step i + 1's upload would queue behind step i's
    # read-back, which waits for step i's kernels), so step i + 1's inputs cross
    # PCIe while step i computes: the way a serving loop feeds the GPU
    in_bytes, out_words = _e2e_sizes(w.R, w.H, n)
    pin_in = [torch.empty(in_bytes, dtype=torch.uint8).pin_memory() for _ in range(2)]
    for b in range(2):
        pin_in[b][: w.R * w.H * 2].view(torch.bfloat16).view(w.R, w.H).copy_(hidden.cpu())
        pin_in[b][w.R * w.H * 2:].view(torch.int32).view(w.R, 5).copy_(params.cpu())
    pin_out = [torch.empty(out_words, dtype=torch.int32).pin_memory() for _ in range(2)]
    dev_in = [torch.empty(in_bytes, dtype=torch.uint8, device=dev) for _ in range(2)]
    dev_out = [torch.empty(out_words, dtype=torch.int32, device=dev) for _ in range(2)]
    bufs = [_e2e_views(dev_in[b], dev_out[b], w.R, w.H, n) for b in range(2)]
    up_stream = torch.cuda.Stream(dev)
    down_stream = torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]    # inputs of buffer b are on the device
    ev_done = [torch.cuda.Event() for _ in range(2)]  # the step using buffer b has computed
    ev_out = [torch.cuda.Event() for _ in range(2)]   # results of buffer b are on the host

    def e2e_run(first_seed, nsteps, start=None):
        if start is not None:
            up_stream.wait_event(start)  # no copy of the timed steps starts before the clock
            down_stream.wait_event(start)
        for b in range(2):
            ev_out[b].record(down_stream)
        for i in range(nsteps):
            b = i & 1
            hid, prm, res = bufs[b]
            with torch.cuda.stream(up_stream):
                up_stream.wait_event(ev_out[b])  # buffer b's previous step has been read back
                dev_in[b].copy_(pin_in[b], non_blocking=True)
                ev_in[b].record(up_stream)
            stream.wait_event(ev_in[b])
            project(hid, stream)
            sample(prm, first_seed + i, res, stream)
            ev_done[b].record(stream)
            with torch.cuda.stream(down_stream):
                down_stream.wait_event(ev_done[b])
                pin_out[b].copy_(dev_out[b], non_blocking=True)
                ev_out[b].record(down_stream)
        for b in range(2):
            stream.wait_event(ev_out[b])  # every result is on the host

    e2e_run(0, warmup)
    torch.cuda.synchronize()
    _barrier(world)
    e0, e1 = _events(2)
    e0.record(stream)
    e2e_run(3000, steps, e0)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = _max_over_ranks(e0.elapsed_time(e1), world, dev)
    _barrier(world)

    gemm_bytes = w.V * w.H * 2 + w.R * w.H * 2 + w.R * w.V * 4
    gemm_flops = 2.0 * w.R * w.H * w.V
    samp_bytes = _sampler_read_bytes(w, T, k, samp_stats, sms)
    ridge = tf_peak * 1e12 / (hbm_peak * 1e9)
    gemm_hbm = gemm_flops / gemm_bytes < ridge
    gemm_tf = gemm_flops / (gemm_ms / 1e3) / 1e12
    gemm_gbs = gemm_bytes / (gemm_ms / 1e3) / 1e9
    samp_gbs_cold = samp_bytes / (samp_cold_ms / 1e3) / 1e9
    summary = {
        "rows": w.R, "vocab": w.V, "hidden": w.H, "slices": w.S,
        "step_ms": total_ms / steps, "rows_per_s": world * w.R * steps / (total_ms / 1e3),
        "e2e_rows_per_s": world * w.R * steps / (e2e_ms / 1e3),
        "gemm_ms": gemm_ms, "gemm_tflops": gemm_tf, "gemm_hbm_gbs": gemm_gbs,
        "gemm_bound": "hbm" if gemm_hbm else "tensor",
        "gemm_frac": (gemm_gbs / hbm_peak) if gemm_hbm else (gemm_tf / tf_peak),
        "gemm_frac_of": "measured HBM copy GB/s" if gemm_hbm else "measured bf16 burst TF/s",
        "sample_ms_in_step": samp_ms, "sample_ms_cold_l2": samp_cold_ms,
        "sampler_mode": "tile statistics" if tiles else "full rows",
        "sampler_read_bytes": samp_bytes,
        "sampler_hbm_gbs_cold_l2": samp_gbs_cold, "sampler_frac_cold_l2": samp_gbs_cold / hbm_peak,
        "sampler_full_rows_equiv_gbs": w.R * w.V * 4 / (samp_cold_ms / 1e3) / 1e9,
        "sampler_rows_per_s_cold_l2": w.R / (samp_cold_ms / 1e3),
    }
    state = {"samp_in": samp_in, "params": params, "T": T, "k": k, "p": p, "req": req + rank * w.requests,
             "pos": pos, "total_ms": total_ms, "gemm_ms": gemm_ms, "samp_ms": samp_ms, "e2e_ms": e2e_ms,
             "h2d": in_bytes, "d2h": out_words * 4, "gemm_bytes": gemm_bytes, "gemm_flops": gemm_flops,
             "samp_bytes": samp_bytes, "gemm_hbm": gemm_hbm, "out": out, "samp_stats": samp_stats}
    return summary, state


def run_gpu(args, w):
    import vocab_sharded_logits_b200 as vsl
    world, rank, local = _dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks = _peaks()
    hbm_peak, tf_peak, _, peak_kind = peaks

    clocks = ClockSampler(local)
    clocks.start()
    head, st = measure_config(w, dev, world, rank, args.steps, args.warmup, peaks)
    # a timed region shorter than the sampling period still gets samples
    t0 = time.time()
    while clocks.proc is not None and clocks.count() - clocks.skip < 3 and time.time() - t0 < 10:
        for i in range(10):
            vsl.sample(st["samp_in"], st["params"], 5000 + i, w.n_logprobs, out=st["out"])
        torch.cuda.synchronize()

    # the GPU's draw on the headline's logits for the bench-side parity count
    parity_out = vsl.sample(st["samp_in"], st["params"], PARITY_SEED, w.n_logprobs, tile_stats=st["samp_stats"])
    gpu_tokens = parity_out.token_ids.cpu().numpy()
    logits_host = None
    if rank == 0 and world == 1 and not args.skip_cpu:
        logits_host = torch.cat([t.cpu() for t in st["samp_in"]], dim=1).numpy()
    del parity_out

    per_config = {w.name: head}
    if not args.no_per_config:
        for name in PER_CONFIG:
            if name == w.name:
                continue
            torch.cuda.empty_cache()
            per_config[name], _ = measure_config(W.WORKLOADS[name], dev, world, rank, max(5, args.steps // 2),
                                                 max(3, args.warmup), peaks)
    clk = clocks.stop()
    _barrier(world)

    status = vsl.device_error()
    if status != (0, 0):
        print(f"device error word set: {status}", file=sys.stderr)

    # roofline of the step's dominant kernel (a per-kernel event time inside a
    # millisecond-scale region: the burst peaks)
    if st["gemm_ms"] >= st["samp_ms"]:
        if st["gemm_hbm"]:
            roof = {"kernel": "logits_local_kernel", "bound": "hbm",
                    "achieved": st["gemm_bytes"] / (st["gemm_ms"] / 1e3) / 1e9, "peak": hbm_peak, "unit": "GB/s"}
        else:
            roof = {"kernel": "logits_local_kernel", "bound": "tensor",
                    "achieved": st["gemm_flops"] / (st["gemm_ms"] / 1e3) / 1e12, "peak": tf_peak, "unit": "TFLOP/s"}
    else:
        roof = {"kernel": "sample", "bound": "hbm", "achieved": st["samp_bytes"] / (st["samp_ms"] / 1e3) / 1e9,
                "peak": hbm_peak, "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["peak_source"] = peak_kind
    roof["traffic"] = _recorded_traffic(roof["kernel"], w.name)
    samp_roof = {"kernel": "sample", "bound": "hbm", "achieved": head["sampler_hbm_gbs_cold_l2"], "peak": hbm_peak,
                 "unit": "GB/s", "frac": head["sampler_frac_cold_l2"], "peak_source": peak_kind,
                 "timing": "sampler alone, L2 flushed before every rep", "traffic": _recorded_traffic("sample", w.name)}

    line = {
        "metric": METRIC, "value": head["rows_per_s"], "unit": "rows/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": head["step_ms"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": _config(w),
        "roofline": roof, "sampler_roofline": samp_roof,
        "kernels": {"logits_local_ms": st["gemm_ms"], "sample_ms": st["samp_ms"],
                    "sample_cold_l2_ms": head["sample_ms_cold_l2"], "gemm_tflops": head["gemm_tflops"],
                    "sampler_hbm_gbs_cold_l2": head["sampler_hbm_gbs_cold_l2"]},
        "e2e": {"value": head["e2e_rows_per_s"], "unit": "rows/s", "h2d_bytes_per_step": st["h2d"],
                "d2h_bytes_per_step": st["d2h"]},
        "gpu_launches": (1 + vsl.sample_launches(w.R, w.S, w.V_s)) * args.steps,  # projection + sampler kernels
        "clocks": clk, "per_config": per_config, "cpu_baseline": None, "parity": None,
    }
    if logits_host is not None:
        params = (st["T"], st["k"], st["p"], st["req"], st["pos"])
        line["cpu_baseline"], line["parity"] = oracle_baseline(
            logits_host, params, PARITY_SEED, w.n_logprobs,
            f"the {w.name} workload's projection output (R={w.R}, V={w.V})", gpu_tokens=gpu_tokens,
            budget_s=args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def run_sampler_only(args, w):
    """Times ``sample`` alone on the workload's synthetic fp32 logits (the recipe of
    the parity tests), L2 flushed before every rep, clocks sampled; one JSON line."""
    import vocab_sharded_logits_b200 as vsl
    dev = torch.device("cuda", 0)
    hbm_peak, _, _, peak_kind = _peaks()
    logits = W.sampler_logits(w, dev)
    slices = [t.contiguous() for t in torch.tensor_split(logits, w.S, dim=1)]
    del logits
    T, k, p, req, pos = W.row_params(w)
    params = vsl.make_row_params(T, k, p, req, pos, dev)
    stats = vsl.tile_stats(slices) if args.tile_stats else None
    out = vsl.sample(slices, params, 0, w.n_logprobs, tile_stats=stats)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    for i in range(args.warmup):
        vsl.sample(slices, params, i, w.n_logprobs, out=out, tile_stats=stats)
    clocks = ClockSampler(0)
    clocks.start()
    times = []
    t_start = time.time()
    i = 0
    while i < args.steps or (clocks.proc is not None and clocks.count() - clocks.skip < 3
                             and time.time() - t_start < 10):
        flush.fill_(float(i))
        e0, e1 = _events(2)
        e0.record()
        vsl.sample(slices, params, 100 + i, w.n_logprobs, out=out, tile_stats=stats)
        e1.record()
        torch.cuda.synchronize()
        if i < args.steps:
            times.append(e0.elapsed_time(e1))
        i += 1
    clk = clocks.stop()
    ms = statistics.median(times)
    nbytes = _sampler_read_bytes(w, T, k, stats, torch.cuda.get_device_properties(dev).multi_processor_count)
    print(json.dumps({"metric": f"sampler rows/sec ({w.name}, V={w.V}, L2 flushed)", "value": w.R / (ms / 1e3),
                      "unit": "rows/s", "ms": ms, "hbm_gbs": nbytes / (ms / 1e3) / 1e9,
                      "roofline": {"bound": "hbm", "achieved": nbytes / (ms / 1e3) / 1e9, "peak": hbm_peak,
                                   "unit": "GB/s", "frac": nbytes / (ms / 1e3) / 1e9 / hbm_peak,
                                   "peak_source": peak_kind},
                      "clocks": clk, "read_bytes": nbytes,
                      "config": {"workload": w.name, "rows": w.R, "vocab": w.V, "slices": w.S,
                                 "tile_statistics": bool(args.tile_stats)}}), flush=True)
    return 0


def run_gemm_only(args, w):
    """Times ``logits_local`` alone on the workload's bf16 inputs: ``--steps`` event
    pairs around 10 back-to-back launches each (launch overhead hidden), after
    ``--warmup`` launches, clocks sampled; one JSON line (a profiling aid)."""
    import vocab_sharded_logits_b200 as vsl
    dev = torch.device("cuda", 0)
    hbm_peak, tf_peak, _, peak_kind = _peaks()
    hidden, ws = W.gemm_inputs(w, dev)
    out = [torch.empty(w.R, w.V_s, dtype=torch.float32, device=dev) for _ in range(w.S)]
    stats = torch.empty(vsl.tile_stats_shape(w.R, w.S, w.V_s), device=dev) if args.tile_stats else None
    for _ in range(args.warmup):
        vsl.logits_local(hidden, ws, out=out, tile_stats=stats)
    torch.cuda.synchronize()
    clocks = ClockSampler(0)
    clocks.start()
    times = []
    t_start = time.time()
    i = 0
    while i < args.steps or (clocks.proc is not None and clocks.count() - clocks.skip < 3
                             and time.time() - t_start < 10):
        e0, e1 = _events(2)
        e0.record()
        for _ in range(10):
            vsl.logits_local(hidden, ws, out=out, tile_stats=stats)
        e1.record()
        torch.cuda.synchronize()
        if i < args.steps:
            times.append(e0.elapsed_time(e1) / 10)
        i += 1
    clk = clocks.stop()
    ms = statistics.median(times)
    flops = 2.0 * w.R * w.H * w.V
    nbytes = w.V * w.H * 2 + w.R * w.H * 2 + w.R * w.V * 4
    print(json.dumps({"metric": f"logits_local TFLOP/s ({w.name})", "value": flops / ms / 1e9, "unit": "TFLOP/s",
                      "ms": ms, "hbm_gbs": nbytes / (ms / 1e3) / 1e9, "tflops_frac_of_burst": flops / ms / 1e9 / tf_peak,
                      "hbm_frac": nbytes / (ms / 1e3) / 1e9 / hbm_peak, "peak_source": peak_kind, "clocks": clk,
                      "config": {"workload": w.name, "rows": w.R, "hidden": w.H, "vocab": w.V, "slices": w.S,
                                 "tile_statistics": bool(args.tile_stats)}}),
          flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["vsl", "reference"], default="vsl")
    ap.add_argument("--workload", default="large", choices=sorted(W.WORKLOADS))
    ap.add_argument("--reference-rows", type=int, default=2, help="oracle arm: rows per worker process per step")
    ap.add_argument("--cpu-seconds", type=float, default=2.0, help="cpu_baseline: seconds per timed oracle run")
    ap.add_argument("--skip-cpu", action="store_true")
    ap.add_argument("--no-per-config", action="store_true", help="measure the headline workload only")
    ap.add_argument("--sampler-only", action="store_true",
                    help="time the sampler alone on the workload's synthetic logits (profiling aid)")
    ap.add_argument("--tile-stats", action="store_true",
                    help="with --sampler-only: give the sampler the tile statistics of its logits; with "
                         "--gemm-only: the projection also writes them")
    ap.add_argument("--gemm-only", action="store_true",
                    help="time the projection alone, 10 back-to-back launches per timing (profiling aid)")
    args = ap.parse_args()
    w = W.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    if not torch.cuda.is_available():
        print(json.dumps({"error": "no CUDA device"}))
        return 1
    if args.sampler_only:
        return run_sampler_only(args, w)
    if args.gemm_only:
        return run_gemm_only(args, w)
    return run_gpu(args, w)


if __name__ == "__main__":
    sys.exit(main())
