"""Sequence-parallel attention over the ranks of a torch.distributed group.

Page: "compile_graph" (chenyy20.com) §5.  The sequence is split evenly over
the GPUs and every per-token step stays local; only attention needs the
whole sequence.  Two ways to assemble it:
  - Ring: K and V travel around the ranks by point-to-point transfers, one hop
    per rank; every hop computes attention of the local queries against the
    shard in hand and merges it into the running result by log-sum-exp.
  - Ulysses: an all-to-all trades tokens for heads, so each rank holds the
    whole sequence for H/N heads; local attention; an all-to-all trades back.

Each rank holds a contiguous shard of S/N tokens: rank r owns tokens
[r S/N, (r+1) S/N).  Tensors are [S/N, H*128] row-major (head h at columns
h*128), as the block entry points lay them out.  The local operations default
to this library's CUDA kernels (dit_attention with its log-sum-exp,
dit_attention_merge); `attn` and `merge` can be replaced by callables with
the same contracts, which the multi-process CPU tests use to check the
schedules themselves.
"""
from __future__ import annotations


def _cuda_attn(q, k, v, o, lse, H):
    from . import dit_attention
    dit_attention(q, k, v, o, 1, q.shape[0], k.shape[0], H, lse=lse)


def _cuda_merge(o_parts, lse_parts, o, lse, H):
    from . import dit_attention_merge
    dit_attention_merge(o_parts, lse_parts, o, lse, 1, o.shape[0], H)


def _peer(group, r):
    import torch.distributed as dist
    return r if group is None else dist.get_global_rank(group, r)


def ring_attention(q, k, v, out, H, group=None, attn=None, merge=None):
    """out = attention(q, K, V) where K and V are the concatenation of every
    rank's k and v shards.  N - 1 hops: the shard in hand is sent to rank r+1
    and the next one received from rank r-1 while the local attention of the
    shard in hand runs; each hop's result is merged into `out` by log-sum-exp.
    Returns the fp32 log-sum-exp [H, S/N] of the local queries over all keys."""
    import torch
    import torch.distributed as dist
    attn = attn or _cuda_attn
    merge = merge or _cuda_merge
    N = dist.get_world_size(group)
    r = dist.get_rank(group)
    S_loc = q.shape[0]
    kv = torch.stack([k, v])
    buf = torch.empty_like(kv)
    lse = torch.empty((H, S_loc), dtype=torch.float32, device=q.device)
    part = torch.empty_like(out)
    lse_part = torch.empty_like(lse)
    nxt, prv = _peer(group, (r + 1) % N), _peer(group, (r - 1) % N)
    for hop in range(N):
        reqs = []
        if hop < N - 1:
            # one group for the send and the receive: with NCCL, separate calls
            # would queue every rank's send ahead of its receive and wait in a cycle
            reqs = dist.batch_isend_irecv([dist.P2POp(dist.isend, kv, nxt, group),
                                           dist.P2POp(dist.irecv, buf, prv, group)])
        if hop == 0:
            attn(q, kv[0], kv[1], out, lse, H)
        else:
            attn(q, kv[0], kv[1], part, lse_part, H)
            merge([out, part], [lse, lse_part], out, lse, H)
        for req in reqs:
            req.wait()
        if hop < N - 1:
            kv, buf = buf, kv
    return lse


def ulysses_attention(q, k, v, out, H, group=None, attn=None):
    """out = attention(q, K, V) over the whole sequence with heads split across
    ranks: an all-to-all gives rank r all tokens of heads [r H/N, (r+1) H/N),
    attention runs there, and a second all-to-all returns every rank its own
    tokens.  H must be a multiple of the group size."""
    import torch
    import torch.distributed as dist
    attn = attn or _cuda_attn
    N = dist.get_world_size(group)
    if H % N:
        raise ValueError(f"{H} heads do not split over {N} ranks")
    S_loc = q.shape[0]
    Hl = H // N
    w = Hl * 128

    def to_heads(t):  # [S_loc, H*128] -> [S, Hl*128]: this rank's heads, every rank's tokens
        send = t.reshape(S_loc, N, w).transpose(0, 1).contiguous()  # [N, S_loc, w], chunk i -> rank i
        recv = torch.empty_like(send)
        dist.all_to_all_single(recv, send, group=group)
        return recv.reshape(N * S_loc, w)  # rank i's tokens in rank order

    qh, kh, vh = to_heads(q), to_heads(k), to_heads(v)
    oh = torch.empty_like(qh)
    attn(qh, kh, vh, oh, None, Hl)
    send = oh.reshape(N, S_loc, w).contiguous()  # token chunk i -> rank i
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    out.copy_(recv.transpose(0, 1).reshape(S_loc, N * w))  # head group i came from rank i
    return out
