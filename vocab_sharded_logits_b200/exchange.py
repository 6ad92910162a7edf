"""Batch-sharded sampling across ranks: the vocab-sliced projection's exchange.

"Qwen4Exp batch-sharded sampling: inside vLLM PR #61018" (orcarouter.ai blog),
section "batch-sharded sampling in one paragraph": every tensor-parallel rank
computes only its own slice of the vocabulary projection (no gather), the
ranks exchange slices all-to-all so that each holds the full vocabulary of a
1/P share of the rows, each samples its rows, and the (small) results are
gathered.  One process per GPU, ``torch.distributed`` for the collectives
(NCCL on GPUs, gloo for the CPU tests).

Layout: rank p holds ``local_logits`` = its vocab slice p ([R, V_s], fp32) of
all R rows, R a multiple of P.  Rows are split into P consecutive blocks; one
``all_to_all_single`` sends block q of the local slice to rank q, so rank q
receives, from every rank p, slice p of its rows: a [P, R/P, V_s] buffer whose
P parts are exactly the S = P vocab slices ``sample`` takes (token j of part
p has global id p * V_s + j).  No copy is made after the exchange.
"""
import torch
import torch.distributed as dist

__all__ = ["row_block", "exchange_slices", "gather_rows", "batch_sharded_sample"]


def row_block(R, rank, world):
    """The rows rank ``rank`` samples: [rank * R / P, (rank + 1) * R / P)."""
    if R % world != 0:
        raise ValueError(f"rows ({R}) must be a multiple of the ranks ({world})")
    n = R // world
    return slice(rank * n, (rank + 1) * n)


def exchange_slices(local_logits, group=None):
    """All-to-all of vocab slices: returns the P vocab slices [R/P, V_s] of this
    rank's rows (views of one received buffer)."""
    world = dist.get_world_size(group)
    R, V_s = local_logits.shape
    row_block(R, 0, world)
    if not local_logits.is_contiguous():
        raise ValueError("local_logits must be contiguous")
    recv = torch.empty_like(local_logits)
    dist.all_to_all_single(recv, local_logits, group=group)
    return list(recv.view(world, R // world, V_s).unbind(0))


def gather_rows(x, group=None):
    """All-gather of per-rank row blocks along dimension 0."""
    world = dist.get_world_size(group)
    x = x.contiguous()
    out = torch.empty((world * x.shape[0],) + tuple(x.shape[1:]), dtype=x.dtype, device=x.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(out, x, group=group)
    else:
        dist.all_gather(list(out.chunk(world)), x, group=group)
    return out


def batch_sharded_sample(local_logits, params, seed, n_logprobs, group=None, sampler=None):
    """Samples all R rows with the work split by rows across the ranks.

    local_logits: this rank's vocab slice of every row, [R, V_s] (e.g. the one
    slice ``logits_local`` computes on this rank); params: the row parameters of
    all R rows ([R, 5], ``make_row_params``); every rank passes the same seed.
    ``sampler(slices, params, seed, n_logprobs)`` samples rows held as vocab
    slices (default: this package's ``sample``).  Returns the outputs of all R
    rows on every rank (token ids, token logprobs, top-n ids / logprobs, flags).
    """
    if sampler is None:
        from . import sample as sampler
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    rows = row_block(local_logits.shape[0], rank, world)
    slices = exchange_slices(local_logits, group)
    res = sampler(slices, params[rows].contiguous(), seed, n_logprobs)
    parts = [res.token_ids, res.token_logprob, res.topn_ids.contiguous(), res.topn_logprob.contiguous(),
             res.row_flags]
    gathered = [gather_rows(t, group) for t in parts]
    return type(res)(*gathered)
