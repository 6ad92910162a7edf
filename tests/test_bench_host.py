"""Host-side logic of bench.py on CPU: the multi-rank timing reduction over a
world-size-2 gloo group, and the reference arm's JSON line."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, _ = bench._dist_setup(world)
    bench._barrier(w)
    got = bench._max_over_ranks(10.0 * (rank + 1), w, "cpu")
    q.put((r, w, got))
    dist.destroy_process_group()


def test_max_over_ranks_gloo_world_size_2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert res == [(0, 2, 20.0), (1, 2, 20.0)]


def test_reference_arm_prints_one_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                          "tiny", "--steps", "2", "--warmup", "1", "--reference-rows", "2"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "rows/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["cpu_baseline"]["nproc"] >= 1 and "cpu_model" in d["cpu_baseline"]


@pytest.mark.parametrize("R,H,n", [(64, 4096, 20), (4, 64, 5), (7, 24, 0)])
def test_e2e_packed_buffers_are_split_without_overlap(R, H, n):
    """The end-to-end leg's packed transfers: the views of hidden, params and the
    five outputs tile the two buffers exactly, with the shapes and dtypes the
    binding checks, and the params block starts 16-byte aligned."""
    import torch
    sys.path.insert(0, ROOT)
    import bench
    in_bytes, out_words = bench._e2e_sizes(R, H, n)
    bi = torch.zeros(in_bytes, dtype=torch.uint8)
    bo = torch.zeros(out_words, dtype=torch.int32)
    hid, prm, res = bench._e2e_views(bi, bo, R, H, n)
    assert hid.dtype == torch.bfloat16 and tuple(hid.shape) == (R, H) and hid.is_contiguous()
    assert prm.dtype == torch.int32 and tuple(prm.shape) == (R, 5) and prm.is_contiguous()
    assert (prm.data_ptr() - bi.data_ptr()) % 16 == 0
    outs = [res.token_ids, res.token_logprob, res.topn_ids, res.topn_logprob, res.row_flags]
    assert [t.dtype for t in outs] == [torch.int32, torch.float32, torch.int32, torch.float32, torch.int32]
    assert [tuple(t.shape) for t in outs] == [(R,), (R,), (R, n), (R, n), (R,)]
    def spans(ts, base):
        return sorted((t.data_ptr() - base, t.data_ptr() - base + t.numel() * t.element_size()) for t in ts)
    for parts, buf in (([hid, prm], bi), (outs, bo)):
        sp = [x for x in spans(parts, buf.data_ptr()) if x[0] != x[1]]
        assert sp[0][0] == 0 and sp[-1][1] == buf.numel() * buf.element_size()
        assert all(a[1] == b[0] for a, b in zip(sp, sp[1:]))


def test_clock_sampler_reads_clocks_and_throttle_reasons(tmp_path):
    """The clocks line of the JSON: median SM clock under load, the max clock and
    every throttle reason seen active, from nvidia-smi's CSV (samples taken
    before the timed steps are skipped)."""
    sys.path.insert(0, ROOT)
    import bench
    csv = tmp_path / "clocks.csv"
    csv.write_text("\n".join([
        "0, 1200, 1965, 150.0, 0x0, Not Active, Not Active, Not Active, Not Active",   # before the steps
        "0, 1965, 1965, 700.5, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1950, 1965, 710.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1935, 1965, 690.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
    ]) + "\n")

    class _Proc:
        def send_signal(self, sig):
            pass

        def wait(self, timeout=None):
            return 0

    c = bench.ClockSampler(0)
    c.proc, c.path, c.skip = _Proc(), str(csv), 1
    got = c.stop()
    assert got == {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}


def test_recorded_traffic_needs_the_sources_it_was_captured_from(monkeypatch, tmp_path):
    """A profile's DRAM bytes are used only while the kernel's sources hash to
    the value recorded beside them."""
    sys.path.insert(0, ROOT)
    import bench
    (tmp_path / "logits_local_kernel_decode.md").write_text(
        "# capture\n"
        f"source_sha256: {bench._source_sha('logits_local_kernel')}\n"
        "traffic_bytes_per_launch: 1253643368\n")
    got = bench._recorded_traffic("logits_local_kernel", "decode", str(tmp_path))
    assert got == 1253643368
    monkeypatch.setattr(bench, "_source_sha", lambda kernel: "0" * 64)
    assert bench._recorded_traffic("logits_local_kernel", "decode", str(tmp_path)) is None
    assert bench._recorded_traffic("logits_local_kernel", "no_such_workload", str(tmp_path)) is None


def test_reference_arm_loads_no_repository_library():
    """The oracle arm imports neither the binding nor libvsl.so: its process maps
    no shared object of this repository."""
    code = ("import sys, runpy; sys.argv = ['bench.py', '--impl', 'reference', '--workload', 'tiny', '--steps', '1', "
            "'--warmup', '0', '--reference-rows', '1']\n"
            "try:\n    runpy.run_path('bench.py', run_name='__main__')\n"
            "except SystemExit as e:\n    assert not e.code, e.code\n"
            "maps = open('/proc/self/maps').read()\n"
            "print('checked')\n"
            "assert 'libvsl' not in maps, 'libvsl mapped'\n"
            "assert 'vocab_sharded_logits_b200' not in sys.modules\n")
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr
    assert "checked" in out.stdout


def test_oracle_timing_harness_matches_the_oracle_on_every_row():
    """The baseline's worker processes run the oracle itself: their tokens equal
    sample_row's on the same rows, in one process and split over workers."""
    import numpy as np
    sys.path.insert(0, ROOT)
    import workloads as W
    from oracle.sampler import sample_row
    from oracle.timing import OracleSampler
    w = W.scaled(W.WORKLOADS["decode"], V=4096, requests=6)
    logits = W.sampler_logits(w, "cpu").numpy()
    T, k, p, req, pos = W.row_params(w)
    want = [sample_row(logits[r], T[r], int(k[r]), p[r], int(req[r]), int(pos[r]), 5, w.n_logprobs).token
            for r in range(w.R)]
    orc = OracleSampler(logits, (T, k, p, req, pos), 5, w.n_logprobs, workers=2)
    try:
        _, one = orc.run(range(w.R), parallel=False)
        orc.start_workers()
        _, many = orc.run(range(w.R), parallel=True)
    finally:
        orc.close()
    assert [t for _, t, _, _, _ in sorted(one)] == want
    assert [t for _, t, _, _, _ in sorted(many)] == want


def test_tile_mode_row_selection():
    """Which rows take the sampler's tile mode in the bench's accounting, and
    when the step requests tile statistics (host logic, no device)."""
    import bench
    import workloads as W
    V = 151936
    T = [0.0, 0.8, 0.8, 0.8, 1.0]
    k = [0, 40, 0, 2000, V]
    assert bench._tile_rows(T, k, V).tolist() == [True, True, False, False, False]
    sms = 148
    for name, want in [("decode", True), ("spec", True), ("large", True), ("peaked", True), ("tiny", True)]:
        w = W.WORKLOADS[name]
        Tw, kw, _, _, _ = W.row_params(w)
        assert bench._uses_tiles(w, Tw, kw, sms) == want, name
    # a small batch of top-k-off rows only: the records would go unused
    w = W.scaled(W.WORKLOADS["large"], requests=4)
    Tw, kw, _, _, _ = W.row_params(w)
    assert not bench._large_batch(w, sms) and not bench._uses_tiles(w, Tw, kw, sms)
    # without records every row reads its V logits
    assert bench._sampler_read_bytes(w, Tw, kw, None, sms) == w.R * w.V * 4
