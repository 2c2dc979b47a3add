"""Context parallelism across GPUs: ring and Ulysses schedules.

The Wave Forcing digest (airadar.tv) compares its Wave Parallelism with the two
standard ways to spread one long attention over several GPUs: Ulysses
(all-to-all from sequence shards to head shards and back) and Ring context
parallelism (K/V blocks passed around a ring, partial results merged).  Both
are built here on ``torch.distributed`` (NCCL over NVLink on GPUs) for the
exchange; every arithmetic step runs in the library's CUDA kernels:
``vdit_attn_fwd`` for each attention and ``vdit_attn_merge`` to fold partial
results through their log-sum-exp.  The exchange and the compute are
separate calls here -- NCCL moves the blocks, the kernels consume them from
local memory.

``attn`` and ``merge`` may be replaced (tests use this to check the
schedules on CPU ranks); by default they are the CUDA entry points and the
functions fail loudly without the built library.

The exchange goes through whatever process group the caller set up: NCCL
moves CUDA tensors directly; a gloo group carries CPU tensors only, so CUDA
tensors are staged through host memory for it (plumbing, no arithmetic).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import binding as vb


# Shards of at most this many keys run the short-key (cross-attention)
# schedule; longer ones the full kernel.  Both compute the same attention.
SHORT_KV = 512


def _default_attn(scale, mask_kind=None, chunk_tokens=0):
    def attn(q, k, v):
        mk = mask_kind
        if mk is None:
            mk = vb.VDIT_MASK_CROSS if k.shape[1] <= SHORT_KV else vb.VDIT_MASK_FULL
        return vb.attention(q, k, v, scale, mk, chunk_tokens)
    return attn


def _default_merge(o_acc, lse_acc, o_part, lse_part, o_out=None):
    B, S, H, D = o_part.shape
    vb.vdit_attn_merge_f32(o_acc, lse_acc, o_part, lse_part, o_out, B, H, S, D)


def _staged(t, group):
    """True when `t` must travel through host memory: a CUDA tensor on a gloo group."""
    return t.is_cuda and dist.get_backend(group) == "gloo"


def ring_attention(q, k, v, group=None, scale=None, attn=None, merge=None):
    """Full (bidirectional) attention of this rank's queries over every rank's keys.

    q: this rank's query shard [B, Sq_local, H, D]; k, v: this rank's K/V shard
    [B, Skv_local, H, D], the same shape on every rank.  At step s rank r holds
    the K/V shard of rank (r - s) mod N; while it attends to that shard it is
    already sending it to rank r + 1 and receiving the next one from rank r - 1.
    The running result is kept in fp32 (``vdit_attn_merge_f32``) and rounded
    to bf16 once, by the last fold.
    Returns (o, lse) for this rank's queries over all N * Skv_local keys.
    """
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if scale is None:
        scale = 1.0 / float(q.shape[-1]) ** 0.5
    attn = attn or _default_attn(scale)
    merge = merge or _default_merge
    if world == 1:
        return attn(q, k.contiguous(), v.contiguous())
    nxt = dist.get_global_rank(group, (rank + 1) % world) if group is not None else (rank + 1) % world
    prv = dist.get_global_rank(group, (rank - 1) % world) if group is not None else (rank - 1) % world
    cur_k, cur_v = k.contiguous(), v.contiguous()
    staged = _staged(cur_k, group)
    B, Sq, H, D = q.shape
    acc_dtype = torch.float32 if q.dtype == torch.bfloat16 else q.dtype
    o_acc = torch.zeros((B, Sq, H, D), dtype=acc_dtype, device=q.device)
    lse_acc = torch.full((B, H, Sq), float("-inf"), dtype=acc_dtype, device=q.device)
    o_out = torch.empty_like(q)
    for step in range(world):
        reqs = []
        if step + 1 < world:
            sk, sv = (cur_k.cpu(), cur_v.cpu()) if staged else (cur_k, cur_v)
            nk, nv = torch.empty_like(sk), torch.empty_like(sv)
            ops = [dist.P2POp(dist.isend, sk, nxt, group), dist.P2POp(dist.isend, sv, nxt, group),
                   dist.P2POp(dist.irecv, nk, prv, group), dist.P2POp(dist.irecv, nv, prv, group)]
            reqs = dist.batch_isend_irecv(ops)
        o_part, lse_part = attn(q, cur_k, cur_v)
        merge(o_acc, lse_acc, o_part, lse_part, o_out if step + 1 == world else None)
        for r in reqs:
            r.wait()
        if step + 1 < world:
            cur_k, cur_v = (nk.to(q.device), nv.to(q.device)) if staged else (nk, nv)
    return o_out, lse_acc


def _all_to_all(recv, send, group):
    if _staged(send, group):
        host = torch.empty(recv.shape, dtype=recv.dtype)
        dist.all_to_all_single(host, send.cpu(), group=group)
        recv.copy_(host)
    else:
        dist.all_to_all_single(recv, send, group=group)


def seq_to_head_shards(x, group=None):
    """[B, S/N, H, D] sequence shard -> [B, S, H/N, D] head shard (all-to-all)."""
    world = dist.get_world_size(group)
    B, s, H, D = x.shape
    if H % world:
        raise ValueError("heads must divide evenly over the ranks")
    hs = H // world
    send = x.reshape(B, s, world, hs, D).permute(2, 0, 1, 3, 4).contiguous()  # [N(dest), B, s, hs, D]
    recv = torch.empty_like(send)                                              # [N(src seq chunk), ...]
    _all_to_all(recv, send, group)
    return recv.permute(1, 0, 2, 3, 4).reshape(B, world * s, hs, D).contiguous()


def head_to_seq_shards(x, group=None):
    """[B, S, H/N, D] head shard -> [B, S/N, H, D] sequence shard (all-to-all)."""
    world = dist.get_world_size(group)
    B, S, hs, D = x.shape
    if S % world:
        raise ValueError("the sequence must divide evenly over the ranks")
    s = S // world
    send = x.reshape(B, world, s, hs, D).permute(1, 0, 2, 3, 4).contiguous()  # [N(dest seq chunk), B, s, hs, D]
    recv = torch.empty_like(send)                                             # [N(src head group), ...]
    _all_to_all(recv, send, group)
    return recv.permute(1, 2, 0, 3, 4).reshape(B, s, world * hs, D).contiguous()


def ulysses_attention(q, k, v, group=None, scale=None, mask_kind=vb.VDIT_MASK_FULL, chunk_tokens=0, attn=None):
    """Attention over sequence-sharded q, k, v ([B, S/N, H, D] each) by head sharding.

    Two all-to-alls bring each rank all S tokens of H/N heads; the attention
    then runs locally (any mask kind, since every rank sees whole sequences),
    and the output goes back to sequence shards.  Returns (o [B, S/N, H, D],
    lse [B, H/N, S] for this rank's heads).
    """
    if scale is None:
        scale = 1.0 / float(q.shape[-1]) ** 0.5
    attn = attn or _default_attn(scale, mask_kind, chunk_tokens)
    qh, kh, vh = (seq_to_head_shards(t, group) for t in (q, k, v))
    o, lse = attn(qh, kh, vh)
    return head_to_seq_shards(o, group), lse
