"""Timing harness of the sampler oracle for the CPU baseline (test infrastructure).

Only ``bench.py`` (its ``cpu_baseline`` leg and ``--impl reference``) uses this
module.  It runs ``oracle.sampler.sample_row``, as it stands, over rows of one
float32 logits matrix in a temporary .npy file that every process maps
read-only: in the calling process (one
thread), or in one worker process per core (each started as a fresh
interpreter that imports only numpy and the oracle, limited to one thread),
the rows split evenly between them.  Wall-clock time of each run, median of
several runs.  A worker that dies ends the run with an error, never a wait.
"""
import json
import os
import shutil
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

_ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


class _Rows:
    """The logits and parameters one process samples from."""

    def __init__(self, path, params, seed, n_logprobs):
        self.logits = np.load(path, mmap_mode="r")
        self.params = [np.asarray(a) for a in params]
        self.seed = seed
        self.n = n_logprobs

    def sample(self, rows):
        from .sampler import sample_row
        T, k, p, req, pos = self.params
        out = []
        for r in rows:
            o = sample_row(np.asarray(self.logits[r]), T[r], int(k[r]), p[r], int(req[r]), int(pos[r]),
                           self.seed, self.n)
            out.append([int(r), int(o.token), bool(o.near_tie), bool(o.cut_tie), int(o.flags)])
        return out


def _serve():
    """Worker loop: a set-up line, then one line of row ids per task, one reply line each."""
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:
        pass
    setup = json.loads(sys.stdin.readline())
    rows = _Rows(setup["path"], setup["params"], setup["seed"], setup["n"])
    print(json.dumps({"ready": True}), flush=True)
    for line in sys.stdin:
        task = json.loads(line)
        print(json.dumps(rows.sample(task)), flush=True)


def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


class OracleSampler:
    """Times the sampler oracle on rows of ``logits`` (float32 [R, V]) with per-row
    ``params`` = (T, k, p, request_id, position) arrays, draw ``seed``."""

    def __init__(self, logits, params, seed, n_logprobs, workers=None):
        self.dir = tempfile.mkdtemp(prefix="vsl_oracle_")
        self.path = os.path.join(self.dir, "logits.npy")
        np.save(self.path, np.ascontiguousarray(logits, dtype=np.float32))
        self.params = [np.asarray(a).tolist() for a in params]
        self.seed = int(seed)
        self.n = int(n_logprobs)
        self.workers = workers or os.cpu_count() or 1
        self.procs = []
        self.local = _Rows(self.path, params, self.seed, self.n)

    def start_workers(self):
        """Starts one worker process per core and waits until each has attached."""
        env = dict(os.environ, OMP_NUM_THREADS="1", OPENBLAS_NUM_THREADS="1", MKL_NUM_THREADS="1",
                   PYTHONPATH=_ROOT + os.pathsep + os.environ.get("PYTHONPATH", ""))
        setup = json.dumps({"path": self.path, "params": self.params, "seed": self.seed, "n": self.n})
        for _ in range(self.workers):
            p = subprocess.Popen([sys.executable, "-c", "from oracle.timing import _serve; _serve()"], cwd=_ROOT,
                                 env=env, stdin=subprocess.PIPE, stdout=subprocess.PIPE, text=True)
            p.stdin.write(setup + "\n")
            p.stdin.flush()
            self.procs.append(p)
        for p in self.procs:
            self._reply(p)

    @staticmethod
    def _reply(p):
        line = p.stdout.readline()
        if not line:
            raise RuntimeError(f"oracle worker {p.pid} exited (status {p.poll()})")
        return json.loads(line)

    def run(self, rows, parallel):
        """Samples ``rows``; returns (seconds, results [row, token, near_tie, cut_tie, flags])."""
        rows = [int(r) for r in rows]
        t0 = time.perf_counter()
        if parallel:
            k = len(self.procs)
            for i, p in enumerate(self.procs):
                p.stdin.write(json.dumps(rows[i::k]) + "\n")
                p.stdin.flush()
            res = [x for p in self.procs for x in self._reply(p)]
        else:
            res = self.local.sample(rows)
        return time.perf_counter() - t0, res

    def median_rate(self, rows, parallel, reps=5):
        """(rows per second of the median run, its seconds, the last run's results)."""
        times, res = [], []
        for _ in range(reps):
            t, res = self.run(rows, parallel)
            times.append(t)
        med = statistics.median(times)
        return len(rows) / med, med, res

    def close(self):
        for p in self.procs:
            try:
                p.stdin.close()
                p.wait(timeout=10)
            except Exception:
                p.kill()
        self.procs = []
        self.local = None
        shutil.rmtree(self.dir, ignore_errors=True)
