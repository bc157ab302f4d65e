"""Context-parallel attention: one sequence sharded along its length over the
ranks of a process group, K/V shards passed round a ring.

The sequence's N positions are cut into chunks; every rank holds the Q, K
and V rows of its chunks.  Each rank's queries must see the keys of every
rank, so the K/V shards travel round the ring (each step sends the shard in
hand to rank r+1 and receives the next one from rank r-1) while the rank
computes the attention of its queries against the shard in hand.  That is
the ring-attention pattern the page lefilia.fr (news digest, mKernel item)
lists among fused multi-GPU kernels.  Each step's result is a partial over a
disjoint key set, and the partials are merged with the LSE rule of
``attn_combine``, the common scale the online softmax keeps between tiles
(page lecompute.fr/kernel-perf/flashattention-4-limites-calcul-matriciel,
section "Deplacer une partie des exponentielles").

Layouts:
  * ``contiguous``: rank r holds positions [r*S, (r+1)*S);
  * ``zigzag``: the sequence is cut into 2W chunks of S/2 and rank r holds
    chunks r and 2W-1-r, so under the causal mask every rank has the same
    amount of work.

The schedule (which chunk pairs to compute at each ring step, with which
causal offset) is plain host logic in :func:`ring_schedule`; the attention
of a chunk pair runs in ``attn_fwd_chunk`` (fp32 output) and the merge in
``attn_combine``.  The ``partial`` and ``merge`` arguments exist so that the
ring logic can be exercised with other implementations of those two steps
(the CPU tests pass the oracle's); the default is the CUDA path.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import _abi

__all__ = ["Chunk", "PairTask", "chunks_of", "ring_schedule", "ring_attention",
           "ring_attention_local"]


@dataclass(frozen=True)
class Chunk:
    """A run of positions: the rows [local, local + length) of a rank's
    shard hold sequence positions [start, start + length)."""
    start: int
    length: int
    local: int


@dataclass(frozen=True)
class PairTask:
    """Attention of one query chunk against one key chunk of the shard in
    hand.  ``causal``: key j (in the key chunk) visible to query i (in the
    query chunk) iff j <= i + delta; otherwise every key is visible."""
    q: Chunk
    k: Chunk
    causal: bool
    delta: int


def chunks_of(rank: int, world: int, n_local: int, layout: str):
    """The chunks of rank ``rank`` when every rank holds ``n_local`` rows."""
    if layout == "contiguous":
        return [Chunk(rank * n_local, n_local, 0)]
    if layout == "zigzag":
        if n_local % 2:
            raise ValueError("zigzag needs an even local length")
        h = n_local // 2
        return [Chunk(rank * h, h, 0), Chunk((2 * world - 1 - rank) * h, h, h)]
    raise ValueError(f"unknown layout {layout!r}")


def pair_task(qc: Chunk, kc: Chunk, causal: bool):
    """The task for one chunk pair, or None when no query sees any key."""
    if not causal:
        return PairTask(qc, kc, False, 0)
    last_q = qc.start + qc.length - 1
    if kc.start > last_q:
        return None                                   # every key is in the future
    if kc.start + kc.length - 1 <= qc.start:
        return PairTask(qc, kc, False, 0)             # every key is visible
    return PairTask(qc, kc, True, qc.start - kc.start)


def ring_schedule(rank: int, world: int, n_local: int, layout: str, causal: bool):
    """For each ring step t = 0 .. world-1: the rank whose K/V shard is in
    hand ((rank - t) mod world) and the chunk-pair tasks to compute on it."""
    mine = chunks_of(rank, world, n_local, layout)
    steps = []
    for t in range(world):
        src = (rank - t) % world
        tasks = []
        for qc in mine:
            for kc in chunks_of(src, world, n_local, layout):
                task = pair_task(qc, kc, causal)
                if task is not None:
                    tasks.append(task)
        steps.append((src, tasks))
    return steps


def _cuda_partial(q, k, v, causal, delta, scale):
    return _abi.attn_fwd_chunk(q, k, v, causal, delta, scale, out_dtype=torch.float32)


def _cuda_merge(o_parts, lse_parts, out_dtype):
    return _abi.attn_combine(o_parts, lse_parts, out_dtype=out_dtype)


def _rows(t, c: Chunk):
    return t[:, :, c.local:c.local + c.length].contiguous()


class _Accumulator:
    """Partial results per query chunk, merged at the end."""

    def __init__(self, chunks):
        self.parts = {c: ([], []) for c in chunks}

    def add(self, c: Chunk, o, lse):
        self.parts[c][0].append(o)
        self.parts[c][1].append(lse)

    def result(self, q, merge, out_dtype):
        B, H, n, d = q.shape
        o = torch.zeros((B, H, n, d), dtype=out_dtype, device=q.device)
        lse = torch.full((B, H, n), float("-inf"), dtype=torch.float32, device=q.device)
        for c, (os_, ls_) in self.parts.items():
            if not os_:
                continue                              # the chunk sees no key at all
            oc, lc = merge(torch.stack(os_), torch.stack(ls_), out_dtype)
            o[:, :, c.local:c.local + c.length] = oc.to(out_dtype)
            lse[:, :, c.local:c.local + c.length] = lc.to(torch.float32)
        return o, lse


def ring_attention(q, k, v, causal: bool = True, scale: float | None = None, group=None,
                   layout: str = "zigzag", partial=None, merge=None):
    """Attention of this rank's queries against the whole sharded sequence.

    q, k, v: this rank's shard, [B, H, n_local, d] (k and v may have fewer
    heads, as for attn_fwd_chunk); every rank holds the same n_local.
    Returns (o [B, H, n_local, d] in q's dtype, lse [B, H, n_local] fp32)
    for the local rows.  Every rank takes the same collective steps: world-1
    rounds of one send to rank+1 and one receive from rank-1 (batched P2P),
    each overlapped with the partials on the shard in hand.
    """
    import torch.distributed as dist
    partial = partial or _cuda_partial
    merge = merge or _cuda_merge
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    B, H, n_local, d = q.shape
    if scale is None:
        scale = d ** -0.5
    sched = ring_schedule(rank, world, n_local, layout, causal)
    acc = _Accumulator(chunks_of(rank, world, n_local, layout))
    nxt, prv = (rank + 1) % world, (rank - 1) % world
    g_next = dist.get_global_rank(group, nxt) if group is not None else nxt
    g_prev = dist.get_global_rank(group, prv) if group is not None else prv
    kv = torch.stack([k, v])                          # one message per step
    for t, (src, tasks) in enumerate(sched):
        reqs = []
        if t + 1 < world:
            recv = torch.empty_like(kv)
            ops = [dist.P2POp(dist.isend, kv, g_next, group),
                   dist.P2POp(dist.irecv, recv, g_prev, group)]
            reqs = dist.batch_isend_irecv(ops)
        for task in tasks:
            o_p, l_p = partial(_rows(q, task.q), _rows(kv[0], task.k), _rows(kv[1], task.k),
                               task.causal, task.delta, scale)
            acc.add(task.q, o_p, l_p)
        for r in reqs:
            r.wait()
        if t + 1 < world:
            kv = recv
    return acc.result(q, merge, q.dtype)


def ring_attention_local(q_shards, k_shards, v_shards, causal: bool = True,
                         scale: float | None = None, layout: str = "zigzag", partial=None,
                         merge=None):
    """Every rank's result of :func:`ring_attention`, computed in one process
    from all shards (the same schedule and kernels, no communication): for
    checking the schedule and the kernels' use of it on one device."""
    partial = partial or _cuda_partial
    merge = merge or _cuda_merge
    world = len(q_shards)
    B, H, n_local, d = q_shards[0].shape
    if scale is None:
        scale = d ** -0.5
    out = []
    for rank in range(world):
        acc = _Accumulator(chunks_of(rank, world, n_local, layout))
        for src, tasks in ring_schedule(rank, world, n_local, layout, causal):
            for task in tasks:
                o_p, l_p = partial(_rows(q_shards[rank], task.q), _rows(k_shards[src], task.k),
                                   _rows(v_shards[src], task.k), task.causal, task.delta, scale)
                acc.add(task.q, o_p, l_p)
        out.append(acc.result(q_shards[rank], merge, q_shards[rank].dtype))
    return out
