"""Parity of the tcgen05 vocab-slice projection with the float64 oracle (GPU):
every element at sizes spanning several tiles and ragged edges, sampled
entries at the five configurations' full sizes, exact results on integer
inputs, determinism, and full overwrite of poisoned outputs."""
import numpy as np
import pytest
import torch

import vocab_sharded_logits_b200 as vsl
from oracle.gemm import logits_local as ref_logits, logits_local_entries
import workloads as W
from parity_helpers import LOGIT_TOL

pytestmark = pytest.mark.gpu


def _np(t):
    return t.float().cpu().numpy()


@pytest.mark.parametrize("R,H,S,V_s", [
    (4, 64, 2, 512),        # tiny config
    (1, 64, 1, 4),          # one row, one partial tile
    (3, 136, 3, 132),       # partial K slab, ragged vocab tile
    (17, 512, 2, 1000),     # ragged batch tile (BN = 32)
    (64, 1024, 1, 2052),    # BN = 64
    (100, 256, 2, 260),     # BN = 128
    (300, 320, 1, 388),     # two batch tiles of 256, ragged
])
def test_full_parity_small(cuda_device, R, H, S, V_s):
    g = torch.Generator(device=cuda_device)
    g.manual_seed(R * 1000 + H)
    hidden = torch.randn(R, H, generator=g, device=cuda_device).to(torch.bfloat16)
    ws = [(torch.randn(V_s, H, generator=g, device=cuda_device) * 0.05).to(torch.bfloat16) for _ in range(S)]
    out = vsl.logits_local(hidden, ws)
    torch.cuda.synchronize()
    ref = ref_logits(_np(hidden), [_np(w) for w in ws])
    for o, r in zip(out, ref):
        assert o.shape == (R, V_s)
        err = np.abs(o.cpu().numpy().astype(np.float64) - r).max()
        assert err <= LOGIT_TOL, err


def test_tiny_config(cuda_device):
    w = W.WORKLOADS["tiny"]
    hidden, ws = W.gemm_inputs(w, cuda_device)
    out = vsl.logits_local(hidden, ws)
    torch.cuda.synchronize()
    ref = ref_logits(_np(hidden), [_np(x) for x in ws])
    for o, r in zip(out, ref):
        assert np.abs(o.cpu().numpy() - r).max() <= LOGIT_TOL


def test_integer_inputs_exact(cuda_device):
    g = torch.Generator(device=cuda_device)
    g.manual_seed(3)
    R, H, V_s = 40, 512, 300
    hidden = torch.randint(-3, 4, (R, H), generator=g, device=cuda_device).to(torch.bfloat16)
    ws = [torch.randint(-3, 4, (V_s, H), generator=g, device=cuda_device).to(torch.bfloat16) for _ in range(2)]
    out = vsl.logits_local(hidden, ws)
    torch.cuda.synchronize()
    ref = ref_logits(_np(hidden), [_np(w) for w in ws])
    for o, r in zip(out, ref):
        assert np.array_equal(o.cpu().numpy().astype(np.float64), r)


@pytest.mark.parametrize("name", ["decode", "spec", "large", "peaked", "wide"])
def test_full_size_sampled_entries(cuda_device, name):
    w = W.WORKLOADS[name]
    hidden, ws = W.gemm_inputs(w, cuda_device)
    out = vsl.logits_local(hidden, ws)
    torch.cuda.synchronize()
    rng = np.random.default_rng(w.index)
    h = _np(hidden)
    for s in range(w.S):
        cols = np.sort(rng.choice(w.V_s, 384, replace=False))
        cols[-1] = w.V_s - 1                                     # the ragged last tile
        wsel = _np(ws[s][torch.as_tensor(cols, device=cuda_device)])
        ref = h.astype(np.float64) @ wsel.astype(np.float64).T
        got = out[s][:, torch.as_tensor(cols, device=cuda_device)].cpu().numpy()
        assert np.abs(got - ref).max() <= LOGIT_TOL
        rows = rng.choice(w.R, 2, replace=False)
        full_ref = logits_local_entries(h, _np(ws[s]), rows, np.arange(w.V_s))
        got_rows = out[s][torch.as_tensor(rows, device=cuda_device)].cpu().numpy()
        assert np.abs(got_rows - full_ref).max() <= LOGIT_TOL


def test_deterministic_and_overwrites_poison(cuda_device):
    w = W.scaled(W.WORKLOADS["spec"], V=4 * 4096)
    hidden, ws = W.gemm_inputs(w, cuda_device)
    a = [torch.full((w.R, w.V_s), float("nan"), device=cuda_device) for _ in range(w.S)]
    b = [torch.full((w.R, w.V_s), float("nan"), device=cuda_device) for _ in range(w.S)]
    vsl.logits_local(hidden, ws, out=a)
    vsl.logits_local(hidden, ws, out=b)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert bool(torch.isfinite(x).all())
        assert torch.equal(x, y)
    assert vsl.device_error() == (0, 0)
