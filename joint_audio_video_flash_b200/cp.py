"""Context-parallel attention over the ranks of a process group (one process per GPU).

The LTX-2.5 DiT splits the video sequence over context-parallel ranks, replicates the
audio stream, and merges cross-attention results through an fp32 all-gather of per-rank
softmax statistics ("feat(ltx2): tile-parallel video VAE and the two-stage pipeline",
commit "Onboard Lightricks LTX-2.5"; "LTX-2: replicate audio stream across Ulysses ranks
by default", Description).  Two exchange patterns cover the block's attentions:

* self-attention over a sharded sequence (video self): every rank receives all shards of K
  and V (one broadcast per source rank), computes its own queries' attention over each
  shard as a partial result (fp32 output and base-2 log-sum-exp,
  ``ltxattn_forward_partial``; its own shard first, then each remote shard as soon as it
  has arrived, while the later ones are still in flight) and merges the partials
  (``ltxattn_combine``);
* replicated queries over sharded keys and values (v2a: audio queries, video keys): every
  rank computes the partial over its own shard; the partials and their statistics are
  all-gathered and merged, so every rank ends with the full result.

a2v (video queries over the replicated audio keys) and audio self-attention need no
exchange: they run locally through ``ltxattn.forward``.

Shards are contiguous, equal ranges of ceil(L / world) tokens, rank r holding tokens
[r * Ls, min(L, (r + 1) * Ls)), zero-padded to Ls; a rank whose range is empty contributes
no partial.  The collectives are torch.distributed broadcasts and all-gathers (NCCL between
GPUs); every step of the attention itself runs in the library's kernels (``backend``, which
tests on CPU replace).
"""
from __future__ import annotations

import math


class LibraryBackend:
    """The library's kernels (CUDA tensors)."""

    def partial(self, q, k, v, kv_valid_len, scale, o_part=None, lse=None):
        from . import ltxattn
        return ltxattn.forward_partial(q, k, v, o_part, lse, kv_valid_len=kv_valid_len,
                                       scale=scale)

    def combine(self, o_parts, lses, q_len):
        from . import ltxattn
        return ltxattn.combine(o_parts, lses, q_len)


def shard_len(total: int, world: int) -> int:
    """Tokens per shard (the last shard may hold fewer real tokens, or none)."""
    return -(-int(total) // int(world))


def shard_valid(total: int, world: int, rank: int) -> int:
    """Real tokens in rank's shard."""
    ls = shard_len(total, world)
    return max(0, min(ls, int(total) - rank * ls))


def _gather(t, group, async_op: bool = False):
    """[world, *t.shape] stack of every rank's t (rank order); with async_op, also the
    collective's handle (wait on it before reading other ranks' slices)."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    out = torch.empty((world, *t.shape), dtype=t.dtype, device=t.device)
    work = dist.all_gather(list(out.unbind(0)), t.contiguous(), group=group, async_op=async_op)
    return (out, work) if async_op else out


def _rows_pad(q_len: int) -> int:
    return -(-int(q_len) // 128) * 128


def _post_shards(parts, group):
    """Every rank's shard, one broadcast per source rank, all posted asynchronously in rank
    order (the same order on every rank, as collectives require).  `parts` are this rank's
    tensors of one shard (e.g. its K and V), stacked into slot [rank] of the returned
    [world, len(parts), *shape] buffer; the other slots receive the other ranks' shards.
    Returns the buffer and one work handle per source rank."""
    import torch
    import torch.distributed as dist
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    buf = torch.empty((world, len(parts), *parts[0].shape), dtype=parts[0].dtype,
                      device=parts[0].device)
    for i, t in enumerate(parts):
        buf[rank, i].copy_(t)
    works = []
    for src in range(world):
        g_src = dist.get_global_rank(group, src) if group is not None else src
        works.append(dist.broadcast(buf[src], src=g_src, group=group, async_op=True))
    return buf, works


def self_attention(q_local, k_local, v_local, seq_len: int, group, *, scale: float | None = None,
                   backend=None):
    """Attention of this rank's query shard over the whole sharded sequence.

    q_local, k_local, v_local: [B, Ls, H, D], this rank's shard of a sequence of seq_len
    tokens (zero-padded to Ls = ceil(seq_len / world)).  Returns [B, Ls, H, D]; rows past
    the rank's real tokens are not meaningful.

    The shards travel one broadcast per source rank; this rank's own partial runs first,
    while they are in flight, and the partial over each remote shard is enqueued right
    after that shard's broadcast (in ring order from this rank), so the transfer of later
    shards overlaps the attention over earlier ones.
    """
    import torch
    import torch.distributed as dist
    backend = backend or LibraryBackend()
    world = dist.get_world_size(group)
    batch, ls, heads, d = q_local.shape
    if ls != shard_len(seq_len, world) or k_local.shape != q_local.shape or \
            v_local.shape != q_local.shape:
        raise ValueError(f"shards must be [B, {shard_len(seq_len, world)}, H, D] on every rank")
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    rank = dist.get_rank(group)
    kvb, works = _post_shards((k_local, v_local), group)  # [world, 2, B, Ls, H, D]
    ranks = [r for r in range(world) if shard_valid(seq_len, world, r) > 0]
    rp = _rows_pad(ls)
    o_parts = torch.empty((len(ranks), batch, heads, rp, d), dtype=torch.float32,
                          device=q_local.device)
    lses = torch.empty((len(ranks), batch, heads, rp), dtype=torch.float32,
                       device=q_local.device)
    for s in range(world):
        r = (rank + s) % world
        if r != rank:
            works[r].wait()  # the stream waits for shard r; the host does not block
        if r in ranks:
            i = ranks.index(r)
            k_r, v_r = (k_local, v_local) if r == rank else (kvb[r, 0], kvb[r, 1])
            backend.partial(q_local, k_r, v_r, shard_valid(seq_len, world, r), scale,
                            o_parts[i], lses[i])
    works[rank].wait()  # this rank's own send has read its slot before the buffer goes
    return backend.combine(o_parts, lses, ls)


def cross_attention(q, k_local, v_local, kv_len: int, group, *, scale: float | None = None,
                    backend=None):
    """Replicated queries over keys and values sharded across the ranks (v2a).

    q: [B, Lq, H, D], the same on every rank; k_local, v_local: [B, Ls, H, D], this rank's
    shard of kv_len tokens.  Every rank returns the full result [B, Lq, H, D].
    """
    import torch.distributed as dist
    backend = backend or LibraryBackend()
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    ls = shard_len(kv_len, world)
    if k_local.shape[1] != ls or v_local.shape != k_local.shape:
        raise ValueError(f"key/value shards must hold {ls} tokens on every rank")
    scale = 1.0 / math.sqrt(q.shape[3]) if scale is None else scale
    valid = shard_valid(kv_len, world, rank)
    if valid > 0:
        o_part, lse = backend.partial(q, k_local, v_local, valid, scale)
    else:
        import torch
        batch, q_len, heads, d = q.shape
        rp = _rows_pad(q_len)
        o_part = torch.zeros((batch, heads, rp, d), dtype=torch.float32, device=q.device)
        lse = torch.full((batch, heads, rp), -math.inf, dtype=torch.float32, device=q.device)
    og, lg = _gather(o_part, group), _gather(lse, group)
    ranks = [r for r in range(world) if shard_valid(kv_len, world, r) > 0]
    if len(ranks) < world:
        og, lg = og[ranks].contiguous(), lg[ranks].contiguous()
    return backend.combine(og, lg, q.shape[1])
