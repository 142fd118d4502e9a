"""Ring attention (context parallelism): exact attention over a sequence whose
query, key and value rows are sharded across a ring of ranks.

The sequence of N rows is split into P equal contiguous shards, shard r on
rank r. In step s = 0 .. P-1 rank r holds the key/value shard of rank
(r - s) mod P and attends its own query shard to it with one ``attn_fwd_f32``: the
whole shard without a causal mask or when it lies earlier in the sequence, the
causal diagonal for its own shard, nothing for a later shard under the causal
mask. Each block's (O, LSE) is folded into the rank's running result with
``attn_merge`` (FlashAttention-3 page: attention over parts of the key range
merges by the parts' log-sum-exp, as in its split-K combine and the
RingAttention derivation it refers to). Meanwhile the shard moves one rank on:
a NCCL send to rank r+1 and receive from rank r-1 into this rank's own HBM,
double-buffered and overlapped with the step's attention (the send/receive
pair is issued before the step's kernels and waited for after them).

Every step of the computation runs in the library's CUDA kernels; the
exchange uses torch.distributed point-to-point operations (NCCL on GPUs).
``ring_attention_emulated`` runs the same per-rank steps for P virtual ranks in
one process on one GPU, with the exchange replaced by reading the source
shard directly; it exists to check and time the ring's arithmetic where only
one GPU is available.
"""
from __future__ import annotations

import math

import torch
import torch.distributed as dist

from . import _binding as _b

FULL, DIAG, SKIP = "full", "diag", "skip"


def ring_schedule(rank: int, world: int, causal: bool):
    """[(source rank, kind)] for steps 0 .. world-1 of ``rank``: in step s the
    rank holds the key/value shard of rank (rank - s) mod world; kind is FULL
    (every key visible), DIAG (own shard, causal mask) or SKIP (a later shard
    under the causal mask)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("ring_schedule: need 0 <= rank < world")
    out = []
    for s in range(world):
        src = (rank - s) % world
        if not causal:
            kind = FULL
        elif src == rank:
            kind = DIAG
        elif src < rank:
            kind = FULL
        else:
            kind = SKIP
        out.append((src, kind))
    return out


def ring_exchange(send, recv, group=None):
    """Posts the ring step's point-to-point operations: every tensor of ``send``
    goes to the next rank of ``group``, every tensor of ``recv`` is filled from the
    previous one. Returns the requests; wait on all of them before reading
    ``recv`` or writing ``send``."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    nxt, prv = (rank + 1) % world, (rank - 1) % world
    if group is not None:
        nxt, prv = dist.get_global_rank(group, nxt), dist.get_global_rank(group, prv)
    ops = [dist.P2POp(dist.isend, t, nxt, group) for t in send]
    ops += [dist.P2POp(dist.irecv, t, prv, group) for t in recv]
    return dist.batch_isend_irecv(ops)


class _RankState:
    """The running (O, LSE) of one rank's query shard and its block scratch."""

    def __init__(self, q: torch.Tensor, scale: float):
        B, Hq, n, d = q.shape
        self.q, self.scale = q, scale
        self.o_acc = torch.empty(B, Hq, n, d, dtype=torch.float32, device=q.device)
        self.lse = torch.empty(B, Hq, n, dtype=torch.float32, device=q.device)
        self.o_blk = torch.empty(B, Hq, n, d, dtype=torch.float32, device=q.device)
        self.lse_blk = torch.empty(B, Hq, n, dtype=torch.float32, device=q.device)
        self.merged = 0

    def add(self, k: torch.Tensor, v: torch.Tensor, kind: str, out=None, stream=None):
        """Attends the query shard to one key/value shard and folds the block in;
        with ``out`` (bf16, the query shard's shape) the merged O is written there."""
        if kind == SKIP:
            return
        # the block's O stays fp32 so the result is rounded to bf16 once, at the last merge
        _b.attn_fwd_f32(self.q, k, v, self.o_blk, self.lse_blk, kind == DIAG, self.scale, stream)
        _b.attn_merge(self.o_acc, self.lse, self.o_blk, self.lse_blk, out=out, init=self.merged == 0,
                      stream=stream)
        self.merged += 1


def _check_shards(q, k, v):
    if q.dim() != 4 or k.shape != v.shape or k.dim() != 4:
        raise ValueError("ring attention: q [B,Hq,n,d], k/v [B,Hkv,n,d]")
    if q.shape[0] != k.shape[0] or q.shape[2] != k.shape[2] or q.shape[3] != k.shape[3]:
        raise ValueError("ring attention: query and key/value shards must have the same B, n and d")


def ring_attention(q, k, v, causal: bool = False, scale: float | None = None, group=None):
    """Ring attention over the ranks of ``group`` (default: the whole world).

    q [B, Hq, n, d] and k, v [B, Hkv, n, d] are this rank's shards (rows
    [rank*n, rank*n + n) of a sequence of world*n rows), bf16 CUDA tensors.
    Returns (o [B, Hq, n, d] bf16, lse [B, Hq, n] fp32) for this rank's rows,
    equal to exact attention over the whole sequence (causal: row i sees keys
    j <= i of the whole sequence). k and v are not modified. Kernels run on
    torch's current stream, which the NCCL operations are ordered against.
    """
    _check_shards(q, k, v)
    scale = 1.0 / math.sqrt(q.shape[-1]) if scale is None else float(scale)
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    sched = ring_schedule(rank, world, causal)
    last = max(s for s, (_, kind) in enumerate(sched) if kind != SKIP)
    st = _RankState(q, scale)
    o = torch.empty_like(q)
    landing = [(torch.empty_like(k), torch.empty_like(v)) for _ in range(min(2, world - 1))]
    cur = (k, v)
    for s, (_, kind) in enumerate(sched):
        reqs = []
        if s + 1 < world:
            nxt = landing[s % 2]
            reqs = ring_exchange(list(cur), list(nxt), group)
        st.add(cur[0], cur[1], kind, out=o if s == last else None)
        for r in reqs:
            r.wait()
        if s + 1 < world:
            cur = nxt
    return o, st.lse


def ring_attention_emulated(q, k, v, world: int, causal: bool = False, scale: float | None = None):
    """The ring's per-rank steps for ``world`` virtual ranks in one process.

    q [B, Hq, N, d], k/v [B, Hkv, N, d] hold the whole sequence (N divisible by
    world); rank r's shard is rows [r*N/world, (r+1)*N/world). Each virtual rank
    runs its schedule with the source shard read directly instead of received.
    Returns (o [B, Hq, N, d] bf16, lse [B, Hq, N] fp32)."""
    if world < 1 or q.shape[2] % world != 0:
        raise ValueError("ring_attention_emulated: N must be a multiple of world")
    _check_shards(q, k, v)
    scale = 1.0 / math.sqrt(q.shape[-1]) if scale is None else float(scale)
    n = q.shape[2] // world
    shard = lambda t, r: t[:, :, r * n:(r + 1) * n].contiguous()  # noqa: E731
    ks = [shard(k, r) for r in range(world)]
    vs = [shard(v, r) for r in range(world)]
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    for r in range(world):
        sched = ring_schedule(r, world, causal)
        last = max(s for s, (_, kind) in enumerate(sched) if kind != SKIP)
        st = _RankState(shard(q, r), scale)
        o_r = torch.empty_like(st.q)
        for s, (src, kind) in enumerate(sched):
            st.add(ks[src], vs[src], kind, out=o_r if s == last else None)
        o[:, :, r * n:(r + 1) * n] = o_r
        lse[:, :, r * n:(r + 1) * n] = st.lse
    return o, lse
