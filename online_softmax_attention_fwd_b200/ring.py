"""Context-parallel ring forward: one long sequence's attention spread over the ranks of a group.

The online softmax is a monoid ("Não escreva kernels, derive-os", "Aprofundamento", first paragraph),
so the attention of a query block over all keys is the merge of its attentions over any partition
of the keys. Each rank keeps its query rows and passes key/value shards around a ring: at step s it
holds the shard of rank (r - s) mod W, computes the attention of its queries against it with the
library's forward kernel, and folds the partial result into a running one with ``attn_merge``,
while the next shard is already on its way over NCCL point-to-point (NVLink on one node). No
rank ever holds more than two key/value shards, and no data-path collective other than these ring
transfers is used.

Sharding (zigzag): the sequence is cut into 2 W chunks of equal length and rank r holds chunks r and
2 W - 1 - r of Q, K and V (concatenated in that order along the sequence). Under a causal mask every
rank then does the same amount of work at every step: a query chunk sees a key chunk fully when the
key chunk comes earlier, causally when it is the same chunk, and not at all when it comes later.

This module is host orchestration only: every step of the arithmetic runs in libattn.so kernels
(``fwd`` and ``merge``); torch.distributed moves the shards. The per-step work functions can be
replaced (``attend``, ``fold``) so that the schedule itself can be checked on CPU ranks.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Tuple

import torch
import torch.distributed as dist


def zigzag_chunks(rank: int, world: int) -> Tuple[int, int]:
    """The two sequence chunks (of 2 * world) that rank ``rank`` holds, in order."""
    return rank, 2 * world - 1 - rank


def ring_schedule(rank: int, world: int, causal: bool) -> List[Tuple[int, List[Tuple[int, int, bool]]]]:
    """For each ring step: (source rank of the key/value shard held at that step, list of
    (query chunk slot, key chunk slot, causal) pairs to attend). Slots are 0 / 1 within a shard.
    A pair whose key chunk comes after its query chunk (causal) is left out: it sees no key."""
    steps = []
    qc = zigzag_chunks(rank, world)
    for s in range(world):
        src = (rank - s) % world
        kc = zigzag_chunks(src, world)
        pairs = []
        for qi in range(2):
            for ki in range(2):
                if not causal:
                    pairs.append((qi, ki, False))
                elif kc[ki] < qc[qi]:
                    pairs.append((qi, ki, False))
                elif kc[ki] == qc[qi]:
                    pairs.append((qi, ki, True))
        steps.append((src, pairs))
    return steps


def zigzag_shard(x: torch.Tensor, rank: int, world: int, dim: int = 1) -> torch.Tensor:
    """This rank's zigzag shard of a full-sequence tensor (chunks r and 2W-1-r along ``dim``)."""
    chunks = x.chunk(2 * world, dim=dim)
    a, b = zigzag_chunks(rank, world)
    return torch.cat([chunks[a], chunks[b]], dim=dim).contiguous()


def zigzag_unshard(shards: List[torch.Tensor], dim: int = 1) -> torch.Tensor:
    """The full-sequence tensor from every rank's zigzag shard (inverse of ``zigzag_shard``)."""
    world = len(shards)
    chunks: List[Optional[torch.Tensor]] = [None] * (2 * world)
    for r, sh in enumerate(shards):
        a, b = zigzag_chunks(r, world)
        ca, cb = sh.chunk(2, dim=dim)
        chunks[a], chunks[b] = ca, cb
    return torch.cat(chunks, dim=dim)


def _library_attend(q, k, v, causal, scale):
    from . import _binding
    return _binding.fwd(q, k, v, causal=causal, scale=scale)


def _library_fold(o_acc, lse_acc, o_part, lse_part, o_out):
    from . import _binding
    _binding.merge(o_acc, lse_acc, o_part, lse_part, o_out)


def ring_rank_forward(q: torch.Tensor, kv_at_step: Callable[[int], Tuple[torch.Tensor, torch.Tensor]],
                      rank: int, world: int, causal: bool, scale: float,
                      attend: Callable = _library_attend, fold: Callable = _library_fold):
    """One rank's part of the ring: q [B, 2c, Hq, D] is its zigzag shard; ``kv_at_step(s)`` returns
    the (k, v) shard [B, 2c, Hkv, D] it holds at step s (blocking until it has arrived). Returns
    (O [B, 2c, Hq, D] bf16, lse [B, Hq, 2c] fp32)."""
    B, S2, Hq, D = q.shape
    c = S2 // 2
    qs = (q[:, :c].contiguous(), q[:, c:].contiguous())
    # running results in fp32 (fp64 when the inputs are fp64, as in the CPU schedule checks)
    acc = torch.float64 if q.dtype == torch.float64 else torch.float32
    o_acc = [torch.zeros(B, c, Hq, D, dtype=acc, device=q.device) for _ in range(2)]
    lse_acc = [torch.full((B, Hq, c), float("-inf"), dtype=acc, device=q.device) for _ in range(2)]
    o_out = [torch.zeros(B, c, Hq, D, dtype=q.dtype, device=q.device) for _ in range(2)]
    sched = ring_schedule(rank, world, causal)
    last_pair = {}  # query slot -> the (step, pair) of its last fold, which also writes the bf16 output
    for si, (_, pairs) in enumerate(sched):
        for p in pairs:
            last_pair[p[0]] = (si, p)
    for si, (_, pairs) in enumerate(sched):
        if not pairs:
            kv_at_step(si)  # keep the ring moving even when this step has nothing to attend
            continue
        k, v = kv_at_step(si)
        ks = (k[:, :c].contiguous(), k[:, c:].contiguous())
        vs = (v[:, :c].contiguous(), v[:, c:].contiguous())
        for p in pairs:
            qi, ki, pc = p
            o_p, lse_p = attend(qs[qi], ks[ki], vs[ki], pc, scale)
            fold(o_acc[qi], lse_acc[qi], o_p, lse_p, o_out[qi] if last_pair[qi] == (si, p) else None)
    o = torch.cat(o_out, dim=1)
    lse = torch.cat(lse_acc, dim=2)
    return o, lse


def ring_attention_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool, scale: float,
                       group=None, attend: Callable = _library_attend, fold: Callable = _library_fold):
    """The context-parallel forward on the ranks of ``group`` (default: the world). q [B, 2c, Hq, D],
    k, v [B, 2c, Hkv, D] are this rank's zigzag shards of the full sequence (``zigzag_shard``);
    returns this rank's (O [B, 2c, Hq, D], lse [B, Hq, 2c]). Key/value shards travel around the ring
    with batched point-to-point sends and receives (NCCL on GPUs); the transfer of the next shard
    overlaps the current step's attention."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    nxt = dist.get_global_rank(group, (rank + 1) % world) if group is not None else (rank + 1) % world
    prv = dist.get_global_rank(group, (rank - 1) % world) if group is not None else (rank - 1) % world
    cur = torch.stack([k, v]).contiguous()
    bufs = [cur, torch.empty_like(cur)]
    pending = []

    def post(step):
        # send the shard held at `step` on, receive the one for `step + 1`
        send_buf, recv_buf = bufs[step % 2], bufs[(step + 1) % 2]
        ops = [dist.P2POp(dist.isend, send_buf, nxt, group), dist.P2POp(dist.irecv, recv_buf, prv, group)]
        return dist.batch_isend_irecv(ops)

    def kv_at_step(step):
        if step > 0:
            for r in pending.pop(0):
                r.wait()
        if step + 1 < world:
            pending.append(post(step))
        buf = bufs[step % 2]
        return buf[0], buf[1]

    return ring_rank_forward(q, kv_at_step, rank, world, causal, scale, attend, fold)


def ring_attention_fwd_local(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, world: int, causal: bool,
                             scale: float, attend: Callable = _library_attend, fold: Callable = _library_fold):
    """The ring on one device: every rank's part run in turn, with the shard a rank would hold at
    each step taken directly from the full tensors instead of received. Same schedule, kernels and
    merges as ``ring_attention_fwd``; for checking them on one GPU. Full-sequence q [B, S, Hq, D],
    k, v [B, S, Hkv, D] with S divisible by 2 * world; returns full-sequence (O, lse)."""
    outs, lses = [], []
    for r in range(world):
        qr = zigzag_shard(q, r, world)
        kv = {}

        def kv_at_step(step, r=r):
            src = (r - step) % world
            if src not in kv:
                kv[src] = (zigzag_shard(k, src, world), zigzag_shard(v, src, world))
            return kv[src]

        o, lse = ring_rank_forward(qr, kv_at_step, r, world, causal, scale, attend, fold)
        outs.append(o)
        lses.append(lse)
    return zigzag_unshard(outs, dim=1), zigzag_unshard(lses, dim=2)
