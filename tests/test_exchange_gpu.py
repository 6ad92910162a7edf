"""The batch-sharded exchange on the GPU through NCCL with one rank (the only
size one GPU allows): the all-to-all is then the identity, and batch-sharded
sampling must reproduce the CUDA sampler's outputs on the same rows."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch

import vocab_sharded_logits_b200 as vsl
import workloads as W
from vocab_sharded_logits_b200 import exchange as X

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_one_rank_nccl_reproduces_the_sampler(cuda_device):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=cuda_device)
    try:
        w = W.scaled(W.WORKLOADS["decode"], V=4 * 2048, requests=16)
        logits = W.sampler_logits(w, cuda_device)
        T, k, p, req, pos = W.row_params(w)
        prm = vsl.make_row_params(T, k, p, req, pos, cuda_device)
        ref = vsl.sample([logits.contiguous()], prm, 17, w.n_logprobs)
        got = X.batch_sharded_sample(logits.contiguous(), prm, 17, w.n_logprobs)
        torch.cuda.synchronize()
        for a, b in [(ref.token_ids, got.token_ids), (ref.token_logprob, got.token_logprob),
                     (ref.topn_ids, got.topn_ids), (ref.topn_logprob, got.topn_logprob),
                     (ref.row_flags, got.row_flags)]:
            assert np.array_equal(a.cpu().numpy(), b.cpu().numpy(), equal_nan=True)
    finally:
        dist.destroy_process_group()
