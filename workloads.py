"""Seeded synthetic workloads: the shapes, sizes and value distributions of the
five named configurations, shared by the tests, the bench and the oracle's
baseline leg.

Holds no arithmetic of the method itself: only random inputs and per-row
parameters.  It sits outside the product package so that the oracle's timed
baseline imports neither the binding nor the CUDA library.  Every generator is
seeded: parameters with numpy PCG64 (``data_seed = 1000 + config index``),
tensors with a torch generator on the target device (the same seed gives the
same tensor on the same device type).
"""
from dataclasses import dataclass

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    index: int             # position in the list of configurations
    requests: int
    rows_per_request: int  # speculative tokens + 1
    H: int
    V: int
    S: int
    n_logprobs: int

    @property
    def R(self):
        return self.requests * self.rows_per_request

    @property
    def V_s(self):
        return self.V // self.S

    @property
    def data_seed(self):
        return 1000 + self.index


WORKLOADS = {
    "tiny": Workload("tiny", 0, 4, 1, 64, 1024, 2, 5),
    "decode": Workload("decode", 1, 64, 1, 4096, 151936, 4, 20),
    "spec": Workload("spec", 2, 128, 4, 4096, 151936, 4, 20),
    "large": Workload("large", 3, 256, 8, 5120, 151936, 8, 20),
    "peaked": Workload("peaked", 4, 1024, 1, 4096, 262144, 8, 20),
    # a second vocabulary shape: V = 248,320 over H = 2,560 (the wide vocabulary
    # relative to the hidden size that makes projection sharding pay), decode-like
    # batch and parameters, 8 slices of 31,040
    "wide": Workload("wide", 5, 64, 1, 2560, 248320, 8, 20),
}


def scaled(w, V=None, requests=None, H=None, S=None):
    """A smaller instance of workload ``w`` with the same parameter recipe."""
    V = V or w.V
    S = S or w.S
    return Workload(w.name, w.index, requests or w.requests, w.rows_per_request, H or w.H, V, S, min(w.n_logprobs, V))


def row_params(w, seed_offset=0):
    """Per-row (temperature, top_k, top_p, request_id, position) arrays for workload ``w``."""
    rng = np.random.default_rng(w.data_seed + 7919 * seed_offset)
    nreq, per = w.requests, w.rows_per_request
    base_pos = rng.integers(0, 8192, nreq)
    if w.name == "tiny":
        T = np.full(nreq, 1.0)
        k = np.full(nreq, 50)
        p = np.full(nreq, 0.9)
    elif w.name in ("decode", "wide"):
        T = rng.uniform(0.5, 1.5, nreq)
        k = rng.choice([0, 20, 50], nreq)
        p = rng.uniform(0.8, 1.0, nreq)
    elif w.name == "spec":
        T = np.full(nreq, 0.8)
        k = np.full(nreq, 40)
        p = np.full(nreq, 0.95)
        T[rng.choice(nreq, nreq // 4, replace=False)] = 0.0
    elif w.name == "large":
        T = rng.uniform(0.3, 1.2, nreq)
        p = rng.uniform(0.5, 1.0, nreq)
        k = np.zeros(nreq, np.int64)
    elif w.name == "peaked":
        T = np.full(nreq, 1.0)
        k = np.full(nreq, 1000)
        p = np.full(nreq, 0.99)
    else:
        raise KeyError(w.name)
    rep = lambda a: np.repeat(np.asarray(a), per)
    T = rep(T).astype(np.float32)
    k = rep(k).astype(np.int32)
    p = rep(p).astype(np.float32)
    req = rep(np.arange(nreq)).astype(np.int64)
    pos = (rep(base_pos) + np.tile(np.arange(per), nreq)).astype(np.int64)
    return T, k, p, req, pos


def gemm_inputs(w, device, dtype=torch.bfloat16):
    """hidden [R, H] and S weight slices [V_s, H] (bf16) for workload ``w``."""
    g = torch.Generator(device=device)
    g.manual_seed(w.data_seed)
    w_std = 0.05 if w.name == "tiny" else 0.02
    hidden = torch.randn(w.R, w.H, generator=g, device=device, dtype=torch.float32).to(dtype)
    slices = []
    for _ in range(w.S):
        slices.append((torch.randn(w.V_s, w.H, generator=g, device=device, dtype=torch.float32) * w_std).to(dtype))
    return hidden, slices


def sampler_logits(w, device, seed_offset=0):
    """Synthetic fp32 logits [R, V] with the distribution of workload ``w``.

    tiny / decode / spec / large: N(0, sigma^2) with sigma = std(W) * sqrt(H), the
    spread of hidden . W for N(0, 1) hidden states.  peaked: per row a random
    permutation of a Zipf(1.1) tail, -1.1 * ln(rank + 1), with 1-3 planted
    tokens 12 above the tail's maximum, and about 5% of rows quantised to a
    2^-10 grid (exact and near ties).
    """
    g = torch.Generator(device=device)
    g.manual_seed(w.data_seed * 65537 + seed_offset)
    R, V = w.R, w.V
    if w.name != "peaked":
        sigma = (0.05 if w.name == "tiny" else 0.02) * float(np.sqrt(w.H))
        return torch.randn(R, V, generator=g, device=device, dtype=torch.float32) * sigma
    perm = torch.rand(R, V, generator=g, device=device).argsort(dim=1)
    tail = -1.1 * torch.log(torch.arange(1, V + 1, device=device, dtype=torch.float64))
    l = torch.empty(R, V, device=device, dtype=torch.float32)
    l.scatter_(1, perm, tail.to(torch.float32).expand(R, V).contiguous())
    n_planted = torch.randint(1, 4, (R,), generator=g, device=device)
    planted = torch.randint(0, V, (R, 3), generator=g, device=device)
    for j in range(3):
        rows = torch.nonzero(n_planted > j).flatten()
        l[rows, planted[rows, j]] = 12.0
    quant = torch.rand(R, generator=g, device=device) < 0.05
    if bool(quant.any()):
        l[quant] = torch.round(l[quant] * 1024.0) / 1024.0
    return l


def split_slices(logits, S):
    """Contiguous [R, V_s] slices of a [R, V] tensor (slice s = columns s*V_s ...)."""
    V_s = logits.shape[1] // S
    return [logits[:, s * V_s:(s + 1) * V_s].contiguous() for s in range(S)]
