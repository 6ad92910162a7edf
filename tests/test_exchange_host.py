"""The batch-sharded exchange (vocab_sharded_logits_b200/exchange.py) on CPU
ranks over gloo: the all-to-all's layout (each rank receives every vocab slice
of its row block), batch-sharded sampling equal to sampling every row in one
process (the per-rank sampler is the oracle here: the CUDA sampler needs a
GPU), and a rank that leaves before the exchange ending the other rank's
collective with an error instead of a wait."""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _global_logits(R, V):
    g = torch.Generator().manual_seed(1234)
    return torch.randn(R, V, generator=g) * 1.5


def _params(R):
    rng = np.random.default_rng(5)
    T = rng.uniform(0.5, 1.5, R).astype(np.float32)
    T[::5] = 0.0
    k = rng.choice([0, 3, 10], R).astype(np.int32)
    p = rng.uniform(0.6, 1.0, R).astype(np.float32)
    return T, k, p, np.arange(R) // 2, np.arange(R) % 2 + 7


def oracle_sampler(slices, params, seed, n):
    """Samples rows held as vocab slices with the oracle (CPU test stand-in)."""
    sys.path.insert(0, ROOT)
    import vocab_sharded_logits_b200 as vsl
    from oracle.sampler import sample_row
    logits = torch.cat(slices, dim=1).numpy()
    p = params.numpy()
    T, k, tp = p[:, 0].view(np.float32), p[:, 1], p[:, 2].view(np.float32)
    req, pos = p[:, 3].view(np.uint32), p[:, 4].view(np.uint32)
    out = [sample_row(logits[r], T[r], int(k[r]), tp[r], int(req[r]), int(pos[r]), seed, n) for r in range(len(p))]
    return vsl.SampleResult(torch.tensor([o.token for o in out], dtype=torch.int32),
                            torch.tensor([o.token_logprob for o in out], dtype=torch.float32),
                            torch.tensor(np.stack([o.topn_ids for o in out]), dtype=torch.int32),
                            torch.tensor(np.stack([o.topn_logprob for o in out]), dtype=torch.float32),
                            torch.tensor([o.flags for o in out], dtype=torch.int32))


def _rank(rank, world, port, R, V, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import vocab_sharded_logits_b200 as vsl
    from vocab_sharded_logits_b200 import exchange as X
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    full = _global_logits(R, V)
    V_s = V // world
    local = full[:, rank * V_s:(rank + 1) * V_s].contiguous()
    slices = X.exchange_slices(local)
    rows = X.row_block(R, rank, world)
    got = torch.cat(slices, dim=1)
    layout_ok = bool(torch.equal(got, full[rows]))
    T, k, p, req, pos = _params(R)
    params = vsl.make_row_params(T, k, p, req, pos, "cpu")
    res = X.batch_sharded_sample(local, params, 99, 3, sampler=oracle_sampler)
    q.put((rank, layout_ok, res.token_ids.numpy(), res.token_logprob.numpy(), res.topn_ids.numpy(),
           res.row_flags.numpy()))
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_batch_sharded_sampling_equals_one_process(world):
    R, V = 8, 48
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, R, V, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=240) for _ in range(world)]
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    # the reference: every row sampled in one process on the whole vocabulary
    sys.path.insert(0, ROOT)
    import vocab_sharded_logits_b200 as vsl
    T, k, p, req, pos = _params(R)
    ref = oracle_sampler([_global_logits(R, V)], vsl.make_row_params(T, k, p, req, pos, "cpu"), 99, 3)
    for rank, layout_ok, tok, lp, topn, flags in got:
        assert layout_ok, rank
        assert np.array_equal(tok, ref.token_ids.numpy()), rank
        assert np.allclose(lp, ref.token_logprob.numpy()), rank
        assert np.array_equal(topn, ref.topn_ids.numpy()), rank
        assert np.array_equal(flags, ref.row_flags.numpy()), rank


def _rank_leaves(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    from vocab_sharded_logits_b200 import exchange as X
    import time
    t0 = time.time()
    try:
        dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=10))
        dist.barrier()  # every connection is up: the group has run one step together
        if rank == 1:
            os._exit(3)  # leaves between steps, before the exchange, with nothing in flight
        t0 = time.time()
        X.exchange_slices(torch.zeros(4, 8))
        q.put(("no error", time.time() - t0))
    except Exception as e:  # the collective ends with an error
        if rank == 0:
            q.put((type(e).__name__, time.time() - t0))
    q.close()
    q.join_thread()  # the queue's feeder thread has written the result before the process ends
    os._exit(0)


def test_a_rank_that_leaves_ends_the_exchange_with_an_error():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_leaves, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    kind, secs = q.get(timeout=120)
    for p in procs:
        p.join(60)
    assert kind != "no error"
    assert secs < 60
