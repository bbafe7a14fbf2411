"""Ring (context-parallel) attention forward: the sequence is cut into one shard per rank and the
key/value shards travel around the ranks, so no rank ever holds more than two key/value shards.

Rank r holds queries, keys and values of positions [r*n, (r+1)*n).  In step s it has the
key/value shard of rank (r - s) mod W; it computes its queries' attention over that shard as an
unrounded partial result (``fa_fwd_partial``: fp32 O normalised over the shard, and the shard's
logsumexp) while it passes the shard on to rank r+1 and receives the next one from rank r-1.
After W steps the partials are combined exactly by the logsumexp merge (``fa_merge_partials``),
the associative form of the online-softmax rescale (robocikowo.com "Flash Attention": O <-
rescale(O_prev, m_old, m_new) + ...; chipfoundryservices.com glossary "Online Softmax Trick").
With a causal mask, shard j is entirely visible to the queries of shard r when j < r, is the
diagonal block (causal within itself) when j = r, and is hidden when j > r (skipped: it would
contribute a partial with logsumexp -inf).

``ring_steps`` is the schedule; ``ring_forward`` runs it with torch.distributed point-to-point
transfers (NCCL between GPUs, gloo on CPU) and takes the partial and merge functions as
arguments, so the same schedule drives the CUDA path (``cuda_partial`` / ``cuda_merge``, through
the C ABI) or any other implementation of the two steps.
"""
from __future__ import annotations


def ring_steps(rank: int, world: int, causal: bool):
    """[(step, key shard, mode)] for one rank: mode is "full", "causal" (the diagonal block) or
    "skip" (a shard the rank's queries cannot see)."""
    out = []
    for s in range(world):
        j = (rank - s) % world
        if not causal:
            mode = "full"
        elif j == rank:
            mode = "causal"
        elif j < rank:
            mode = "full"
        else:
            mode = "skip"
        out.append((s, j, mode))
    return out


def ring_forward(q, k, v, causal: bool, scale: float, partial, merge, group=None):
    """O and L of this rank's query shard over the whole sequence.

    q: [B, H, n, d]; k, v: [B, H_kv, n, d] -- this rank's shards of contiguous sequence blocks
    (rank r holds positions r*n .. r*n + n - 1).  ``partial(q, k, v, causal, scale)`` returns an
    unrounded partial result (O_part, L_part) of the queries over one key shard;
    ``merge(parts)`` combines a list of them.  Every rank takes part in every transfer, in the
    same order, whatever its mask skips.
    """
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    kv = torch.stack([k, v]).contiguous()
    nxt = (rank + 1) % world
    prv = (rank - 1) % world
    parts = []
    for (s, j, mode) in ring_steps(rank, world, causal):
        recv = None
        reqs = []
        if s + 1 < world:
            # pass the shard on while computing on it (the receive buffer is a fresh tensor, the
            # send buffer is not written until the transfer has completed)
            recv = torch.empty_like(kv)
            reqs = [dist.isend(kv, dst=dist.get_global_rank(group, nxt) if group else nxt,
                               group=group),
                    dist.irecv(recv, src=dist.get_global_rank(group, prv) if group else prv,
                               group=group)]
        if mode != "skip":
            parts.append(partial(q, kv[0], kv[1], mode == "causal", scale))
        for r_ in reqs:
            r_.wait()
        if recv is not None:
            kv = recv
    return merge(parts)


# ------------------------------------------------------------------------------ CUDA steps
def cuda_partial(q, k, v, causal: bool, scale: float | None = None):
    """(O_part fp32 [B, H, n, d], L_part fp32 [B, H, n]) through fa_fwd_partial."""
    import torch

    from . import _check, _default_scale, _shape, _stream_handle, fa_fwd_partial
    B, H, n, d = _shape(q)
    if k.dim() != 4 or k.shape[0] != B or k.shape[3] != d or k.shape[1] < 1 or H % k.shape[1]:
        raise ValueError("k, v must be [B, H_kv, Nk, d] with H_kv dividing q's H")
    Hkv = int(k.shape[1])
    scale = _default_scale(d) if scale is None else float(scale)
    o = torch.empty((B, H, n, d), dtype=torch.float32, device=q.device)
    lse = torch.empty((B, H, n), dtype=torch.float32, device=q.device)
    _check(fa_fwd_partial(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                          B, H, Hkv, n, k.shape[2], d, causal, scale, _stream_handle(q)))
    return o, lse


def cuda_merge(parts):
    """(O bf16, L fp32) from a list of cuda_partial results through fa_merge_partials."""
    import torch

    from . import _check, _stream_handle, fa_merge_partials
    o_parts = torch.stack([p[0] for p in parts]).contiguous()
    l_parts = torch.stack([p[1] for p in parts]).contiguous()
    B, H, n, d = parts[0][0].shape
    o = torch.empty((B, H, n, d), dtype=torch.bfloat16, device=o_parts.device)
    lse = torch.empty((B, H, n), dtype=torch.float32, device=o_parts.device)
    _check(fa_merge_partials(o_parts.data_ptr(), l_parts.data_ptr(), len(parts), o.data_ptr(),
                             lse.data_ptr(), B * H * n, d, _stream_handle(o)))
    return o, lse
