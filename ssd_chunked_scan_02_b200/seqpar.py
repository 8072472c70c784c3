"""Sequence-parallel SSD forward: one sequence split along L across ranks,
with a single exchange.

"Transformers are SSMs" (CiteArk), what this means: the layer lends itself
to large-scale, model-parallel training.  What makes a split along the
sequence cheap is that the state entering a shard acts on it linearly:

    y_t   = y_t|zero start   + exp(cs_t) h_in C_t        (cs from the shard's first token)
    h_end = h_end|zero start + exp(cs_last) h_in

so rank r (holding the r-th contiguous piece of every sequence of the
batch) runs its shard from a zero state, the ranks all-gather one packed
buffer per rank -- the shard's final state and its total log-decay,
b*H*(P*N + 1) fp32 -- and each rank folds the ranks before it into its
entering state h_in (an exclusive scan) and corrects its y and final state.

This module is host logic only: rank bookkeeping, packing, the all-gather.
The arithmetic runs in the library's kernels (``CudaOps``); the tests swap in
other ops to check this logic on CPU ranks.
"""
from __future__ import annotations

import torch

from . import ssd


class CudaOps:
    """The per-rank steps, on the GPU through the C ABI."""

    @staticmethod
    def forward(x, dt, A, B, C, D, chunk_size):
        return ssd.ssd_chunk_scan_fwd(x, dt, A, B, C, D, chunk_size, return_final_states=True)

    @staticmethod
    def logdecay(dt, A):
        return ssd.ssd_seq_logdecay(dt, A)

    @staticmethod
    def combine(local_final, logdecay, init, rank):
        return ssd.ssd_state_exchange_combine(local_final, logdecay, rank, init_states=init)

    @staticmethod
    def correct(h_in, dt, A, C, y, final):
        ssd.ssd_state_correction_fwd(h_in, dt, A, C, y, final_states=final)


def pack(final, logdecay):
    """One flat fp32 buffer per rank: the final state then the log-decays."""
    return torch.cat([final.reshape(-1), logdecay.reshape(-1)])


def unpack(gathered, shape_final, shape_ld):
    """(R, n) gathered buffers -> local finals (R, b,H,P,N), log-decays (R, b,H)."""
    nf = 1
    for s in shape_final:
        nf *= s
    R = gathered.shape[0]
    return (gathered[:, :nf].reshape(R, *shape_final).contiguous(),
            gathered[:, nf:].reshape(R, *shape_ld).contiguous())


def chunk_scan_fwd_seqpar(x, dt, A, B, C, D, chunk_size, init_states=None, group=None,
                          ops=None, want_global_final=True):
    """This rank's piece of the forward over a sequence split along L.

    x, dt, B, C are this rank's shard (b, L_r, ...) of every sequence; A, D
    and init_states (the state entering the whole sequence, or None) are the
    same on every rank.  Returns (y, shard_final, global_final): the shard's
    outputs and the state after the shard, both as if the whole sequence had
    run on one device, and (if asked) the state after the whole sequence,
    the same on every rank.  Exactly one collective: an all-gather of
    b*H*(P*N + 1) fp32 per rank."""
    import torch.distributed as dist
    ops = ops or CudaOps
    rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    y, fin = ops.forward(x, dt, A, B, C, D, chunk_size)
    ld = ops.logdecay(dt, A)
    mine = pack(fin, ld)
    bufs = [torch.empty_like(mine) for _ in range(world)]
    dist.all_gather(bufs, mine, group=group)
    finals, lds = unpack(torch.stack(bufs), tuple(fin.shape), tuple(ld.shape))
    h_in = ops.combine(finals, lds, init_states, rank)
    ops.correct(h_in, dt, A, C, y, fin)
    g_fin = ops.combine(finals, lds, init_states, world) if want_global_final else None
    return y, fin, g_fin
