"""Ring context parallelism for the prefill: each rank holds one contiguous
block of every sequence's queries and keys, attends to the K/V block it
currently holds, merges that partial result into its running (o, lse)
state, and passes the block to the next rank while the next step computes
(kernbench2 commit message, ADR-0060 (long context): head-parallel prefill
with the KV blocks rotated around the ring and an online-softmax merge per
ring step).

The blocks travel as whole tensors between the ranks' own device memory
(point-to-point sends of the process group, NCCL over NVLink on GPUs, gloo on
CPU); no rank reads another's memory directly.  With causal masking rank r
needs only the blocks 0..r: it attends causally to its own block and in full
to the earlier ones, and a block is forwarded only while a later rank still
needs it (it never wraps from the last rank back to rank 0), which halves
the transfers.  Every step is one call of the single-GPU path:
fa_attention_fwd_acc merges the step's result into an fp32 accumulator in
the kernel's epilogue and writes the final output on the last step.
Sliding windows are not supported here.

The per-step computation is injectable so the schedule can run anywhere:
tests on CPU pass a reference implementation.
"""
from __future__ import annotations

from typing import Callable, Iterable, Optional, Sequence, Tuple


def _gpu_step(q, k, v, acc, *, hq, hkv, causal, scale, first, last, epilogue):
    import torch

    from . import fa
    if acc is None:
        acc = (torch.empty(q.shape, dtype=torch.float32, device=q.device),
               torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device))
    out = fa.attention_fwd_acc(q, k, v, acc[0], acc[1], hq=hq, hkv=hkv, causal=causal, scale=scale,
                               first=first, last=last, epilogue=epilogue)
    return acc, out


def attend_blocks(q, blocks: Iterable, *, rank: int, n_blocks: int, hq: int, hkv: int, causal: bool = False,
                  scale: Optional[float] = None, epilogue: Sequence[Tuple[str, float]] = (),
                  step: Optional[Callable] = None):
    """Attention of query block `rank` over the K/V blocks that `blocks`
    yields, in any order: (blk, k, v), blk the index (0..n_blocks-1) of the
    positions the block covers, each index once.  With causal masking blocks
    after `rank` are skipped, block `rank` is attended causally and earlier
    ones in full.  Returns the output block in q's dtype, epilogue applied.

    `step(q, k, v, acc, *, hq, hkv, causal, scale, first, last, epilogue)`
    merges one block's attention into the running state `acc` (None before
    the first) and returns (acc, out), out the final output when `last`."""
    step = step or _gpu_step
    wanted = rank + 1 if causal else n_blocks
    acc, out, seen = None, None, 0
    for blk, k, v in blocks:
        if causal and blk > rank:
            continue
        seen += 1
        acc, out = step(q, k, v, acc, hq=hq, hkv=hkv, causal=causal and blk == rank, scale=scale,
                        first=seen == 1, last=seen == wanted, epilogue=epilogue)
    if seen != wanted:
        raise ValueError(f"query block {rank} saw {seen} of the {wanted} key blocks it attends to")
    return out


def ring_schedule(rank: int, world: int, causal: bool, step: int) -> Tuple[bool, bool]:
    """(send, receive) of `rank` after computing on its block at ring step
    `step`: the held block goes to rank + 1, the next one comes from rank - 1.
    Without the causal mask every block visits every rank.  With it, rank r
    holds block r - s at step s and needs no block after 0, and a block is
    useless past the last rank, so rank r sends at steps s <= r (unless it is
    the last rank) and receives at steps s < r."""
    if step + 1 >= world:
        return False, False
    if not causal:
        return True, True
    return step <= rank and rank < world - 1, step < rank


def _ring_blocks(k, v, group, rank: int, world: int, causal: bool):
    """Yields (blk, k, v) for the blocks this rank holds in turn; the next
    block is already on its way in while the caller computes on the current
    one, and the wait for it follows the caller's return to the generator."""
    import torch
    import torch.distributed as dist

    nxt = dist.get_global_rank(group, (rank + 1) % world)
    prv = dist.get_global_rank(group, (rank - 1) % world)
    cur_k, cur_v = k.contiguous(), v.contiguous()
    # two receive buffers taken in turn: the one received into at step s was
    # sent on at step s + 1, and that send has completed before step s + 2
    # receives into it again (the caller's own k and v are never written)
    bufs = [None, None]
    for s in range(world):
        send, recv = ring_schedule(rank, world, causal, s)
        ops = []
        if send:
            ops += [dist.P2POp(dist.isend, cur_k, nxt, group=group), dist.P2POp(dist.isend, cur_v, nxt, group=group)]
        if recv:
            if bufs[s % 2] is None:
                bufs[s % 2] = (torch.empty_like(cur_k), torch.empty_like(cur_v))
            rk, rv = bufs[s % 2]
            ops += [dist.P2POp(dist.irecv, rk, prv, group=group), dist.P2POp(dist.irecv, rv, prv, group=group)]
        # the block moves on while this step computes; the transfers go out as
        # one group so that NCCL cannot order a send ahead of the receive its
        # neighbour is blocked on
        reqs = dist.batch_isend_irecv(ops) if ops else []
        yield (rank - s) % world, cur_k, cur_v
        for r in reqs:
            r.wait()
        if recv:
            cur_k, cur_v = bufs[s % 2]


def ring_attention_fwd(q, k, v, *, hq: int, hkv: int, causal: bool = False, scale: Optional[float] = None,
                       epilogue: Sequence[Tuple[str, float]] = (), group=None, step: Optional[Callable] = None):
    """Attention of this rank's query block over the keys of every rank.

    q [B*hq, S_r, d], k/v [B*hkv, S_r, d]: this rank's block of positions
    [r*S_r, (r+1)*S_r) of each sequence (every rank holds the same S_r).
    `group` is a torch.distributed process group (None: this process is the
    whole ring).  Returns this rank's output block [B*hq, S_r, d] in q's
    dtype, after the epilogue.  The caller's k and v are sent, never written.
    """
    import torch.distributed as dist

    if group is None:
        return attend_blocks(q, [(0, k, v)], rank=0, n_blocks=1, hq=hq, hkv=hkv, causal=causal, scale=scale,
                             epilogue=epilogue, step=step)
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    return attend_blocks(q, _ring_blocks(k, v, group, rank, world, causal), rank=rank, n_blocks=world, hq=hq,
                         hkv=hkv, causal=causal, scale=scale, epilogue=epilogue, step=step)
