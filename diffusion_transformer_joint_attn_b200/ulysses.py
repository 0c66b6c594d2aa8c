"""Sequence-parallel joint attention over several GPUs (Ulysses), with an
optional split of the batch between GPU groups (classifier-free guidance:
the conditional and unconditional items on different groups).

The pages scale FLUX 3 Klein to 8 B200 by putting the positive and negative
CFG branches on separate GPU groups and splitting the sequence with Ulysses
inside a group (scopeai.cc FLUX 3 Klein story, section on multi-GPU and
deployment; bpdata.com "FLUX 3 Image Klein optimalizálása", section on the
detailed optimisation steps; kinachrichten.com "NVIDIA meldet bis zu
4,45-fach ...", multi-GPU section).  Between the
projections, every rank holds a contiguous slice of the tokens of all heads;
attention needs every token of a head.  Ulysses therefore exchanges, once
before and once after the attention call, which dimension is sharded:

    q, k, v  [B, H, N/P, D]  --all-to-all-->  [B, H/P, N, D]
    attention of the local H/P heads over all N tokens (dit_attn_forward)
    O        [B, H/P, N, D]  --all-to-all-->  [B, H, N/P, D]   (LSE likewise)

Rank r of a group of P holds tokens r*N/P .. (r+1)*N/P - 1 and, in between,
heads r*H/P .. (r+1)*H/P - 1.  The rotary tables cover all N tokens (the
positions of a token do not depend on the rank that holds it).  N and H must
be divisible by P.  The exchanges are NCCL all-to-alls over the group's
process group; the attention of the local heads is the library's kernel,
unless a test passes its own `attn` callable.

With head_groups = G > 1 the exchanges are pipelined per group of heads:
each rank's H/P heads form G groups of H/(P G); the q, k, v all-to-all of
every group is started at once (asynchronous, in group order on the
communicator's stream), the attention of group g waits only for group g's
exchange, and group g's O / LSE exchange starts as soon as its attention is
queued.  So the input exchange of group g+1 and the output exchange of group
g-1 overlap the attention of group g, and only the first group's input and
the last group's output exchange stay exposed.
"""
from __future__ import annotations

from typing import Callable, Optional

import torch
import torch.distributed as dist


def _group_size(group) -> int:
    """Ranks in `group` (the default group if None); 1 without an initialised
    process group, where the exchanges are the identity."""
    if group is None and not (dist.is_available() and dist.is_initialized()):
        return 1
    return dist.get_world_size(group) if group is not None else dist.get_world_size()


def seq_to_head(x: torch.Tensor, group=None) -> torch.Tensor:
    """[B, H, N/P, ...] token shard of every head -> [B, H/P, N, ...] every
    token of this rank's heads."""
    P = _group_size(group)
    B, H, Ns = x.shape[:3]
    rest = x.shape[3:]
    if H % P != 0:
        raise ValueError("the head count %d is not divisible by the group size %d" % (H, P))
    if P == 1:
        return x
    # send chunk p (heads of rank p) to rank p: [P, B, H/P, Ns, ...]
    send = x.reshape(B, P, H // P, Ns, *rest).transpose(0, 1).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    # recv[p] holds rank p's token slice of our heads: tokens in rank order
    return recv.permute(1, 2, 0, 3, *range(4, 4 + len(rest))).reshape(B, H // P, P * Ns, *rest).contiguous()


def head_to_seq(x: torch.Tensor, group=None) -> torch.Tensor:
    """[B, H/P, N, ...] every token of this rank's heads -> [B, H, N/P, ...]
    this rank's tokens of every head (the inverse of seq_to_head)."""
    P = _group_size(group)
    B, Hl, N = x.shape[:3]
    rest = x.shape[3:]
    if N % P != 0:
        raise ValueError("the token count %d is not divisible by the group size %d" % (N, P))
    if P == 1:
        return x
    Ns = N // P
    # send token slice p to rank p: [P, B, H/P, Ns, ...]
    send = x.reshape(B, Hl, P, Ns, *rest).permute(2, 0, 1, 3, *range(4, 4 + len(rest))).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    # recv[p] holds our token slice of rank p's heads: heads in rank order
    return recv.transpose(0, 1).reshape(B, P * Hl, Ns, *rest).contiguous()


def _library_attention(q, k, v, rope_cos, rope_sin, n_txt: int, out_f32: bool, with_lse: bool):
    """The library's attention of the local heads: K rotated and V converted
    once (dit_attn_prepare_kv), then the forward on the prepared operands."""
    from . import dit_attn_prepare_kv, forward
    if rope_cos is None:
        return forward(q, k, v, None, None, n_txt=n_txt, out_f32=out_f32, with_lse=with_lse)
    k_rot = torch.empty_like(k)
    v_f16 = torch.empty(v.shape, dtype=torch.float16, device=v.device)
    dit_attn_prepare_kv(k, v, rope_cos, rope_sin, k_rot, v_f16)
    return forward(q, k_rot, v_f16, rope_cos, rope_sin, n_txt=n_txt, out_f32=out_f32, with_lse=with_lse,
                   k_rotated=True, v_f16=True)


def _heads_of_group(H: int, P: int, G: int, g: int) -> torch.Tensor:
    """Indices of the heads group g carries to each of the P ranks, in rank
    order: rank p's heads p H/P + g H/(P G) + [0, H/(P G))."""
    Hg = H // (P * G)
    return torch.tensor([p * (H // P) + g * Hg + i for p in range(P) for i in range(Hg)], dtype=torch.long)


def _exchange_in(q, k, v, heads, P, group):
    """Start the all-to-all of one head group: every rank sends its token
    shard of rank p's heads of the group to rank p.  Returns (recv, work)."""
    B, _, Ns, D = q.shape
    Hg = heads.numel() // P
    send = torch.stack([t.index_select(1, heads.to(t.device)).reshape(B, P, Hg, Ns, D).transpose(0, 1)
                        for t in (q, k, v)], dim=1).contiguous()            # [P, 3, B, Hg, Ns, D]
    recv = torch.empty_like(send)
    return recv, dist.all_to_all_single(recv, send, group=group, async_op=True)


def _exchange_out(x, P, group):
    """Start the all-to-all that returns one group's result [B, Hg, N, ...]
    to the ranks that hold its tokens.  Returns (recv [P, B, Hg, Ns, ...], work)."""
    B, Hg, N = x.shape[:3]
    rest = x.shape[3:]
    send = x.reshape(B, Hg, P, N // P, *rest).permute(2, 0, 1, 3, *range(4, 4 + len(rest))).contiguous()
    recv = torch.empty_like(send)
    return recv, dist.all_to_all_single(recv, send, group=group, async_op=True)


def _ulysses_grouped(q, k, v, rope_cos, rope_sin, n_txt, group, out_f32, with_lse, attn, P, G):
    B, H, Ns, D = q.shape
    Hl, Hg, N = H // P, H // (P * G), Ns * P
    heads = [_heads_of_group(H, P, G, g) for g in range(G)]
    incoming = [_exchange_in(q, k, v, heads[g], P, group) for g in range(G)]
    outgoing = []
    for g in range(G):
        recv, work = incoming[g]
        work.wait()
        # recv[p]: rank p's token shard of this rank's group-g heads -> [3, B, Hg, N, D]
        qkv = recv.permute(1, 2, 3, 0, 4, 5).reshape(3, B, Hg, N, D)
        out, lse = attn(qkv[0].contiguous(), qkv[1].contiguous(), qkv[2].contiguous(), rope_cos, rope_sin, n_txt,
                        out_f32, with_lse)
        outgoing.append((_exchange_out(out, P, group), _exchange_out(lse, P, group) if lse is not None else None))
    out_full = None
    lse_full = None
    for g, ((o_recv, o_work), lse_ex) in enumerate(outgoing):
        o_work.wait()
        if out_full is None:
            out_full = torch.empty((B, H, Ns, D), dtype=o_recv.dtype, device=o_recv.device)
        # o_recv[p]: this rank's tokens of rank p's group-g heads
        out_full[:, heads[g].to(out_full.device)] = o_recv.transpose(0, 1).reshape(B, P * Hg, Ns, D)
        if lse_ex is not None:
            l_recv, l_work = lse_ex
            l_work.wait()
            if lse_full is None:
                lse_full = torch.empty((B, H, Ns), dtype=l_recv.dtype, device=l_recv.device)
            lse_full[:, heads[g].to(lse_full.device)] = l_recv.transpose(0, 1).reshape(B, P * Hg, Ns)
    assert Hl == G * Hg
    return out_full, lse_full


def ulysses_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, rope_cos=None, rope_sin=None,
                      n_txt: int = 0, group=None, out_f32: bool = False, with_lse: bool = True,
                      attn: Optional[Callable] = None, head_groups: int = 1):
    """Joint attention of the token shards q, k, v [B, H, N/P, D] held by the
    P ranks of `group` (rank r: tokens r N/P .. (r+1) N/P - 1).

    rope_cos / rope_sin: the [N, D/2] tables of all N tokens (or None).
    n_txt: text tokens at the start of the full sequence.
    Returns (out [B, H, N/P, D], lse [B, H, N/P] or None) for this rank's
    tokens.  `attn(q, k, v, rope_cos, rope_sin, n_txt, out_f32, with_lse)`
    replaces the library's attention of the local heads (tests use it to run
    the exchange on the CPU).  head_groups: pipeline the exchanges with the
    attention over this many groups of each rank's heads (H must be divisible
    by P * head_groups).
    """
    if q.shape != k.shape or v.shape[:3] != q.shape[:3]:
        raise ValueError("q, k, v must be [B, H, N/P, D] shards of one shape")
    P = _group_size(group)
    N = q.shape[2] * P
    if rope_cos is not None and rope_cos.shape[0] != N:
        raise ValueError("the rotary tables must cover all %d tokens" % N)
    attn = attn or _library_attention
    if head_groups < 1 or q.shape[1] % (P * head_groups) != 0:
        raise ValueError("%d heads cannot form %d groups on each of %d ranks" % (q.shape[1], head_groups, P))
    if head_groups > 1 and P > 1:
        return _ulysses_grouped(q, k, v, rope_cos, rope_sin, n_txt, group, out_f32, with_lse, attn, P, head_groups)
    qh, kh, vh = (seq_to_head(t, group) for t in (q, k, v))
    out, lse = attn(qh, kh, vh, rope_cos, rope_sin, n_txt, out_f32, with_lse)
    out = head_to_seq(out, group)
    if lse is not None:
        lse = head_to_seq(lse.unsqueeze(-1), group).squeeze(-1)
    return out, lse


def cfg_ulysses_groups(world_size: int, cfg_groups: int):
    """Rank lists of the Ulysses groups when `cfg_groups` groups of
    world_size / cfg_groups consecutive ranks each take a share of the batch
    (the CFG branches): [[0 .. P-1], [P .. 2P-1], ...]."""
    if world_size % cfg_groups != 0:
        raise ValueError("%d ranks cannot form %d equal groups" % (world_size, cfg_groups))
    P = world_size // cfg_groups
    return [list(range(g * P, (g + 1) * P)) for g in range(cfg_groups)]


def batch_share(B: int, group_index: int, cfg_groups: int) -> slice:
    """The batch items group `group_index` of `cfg_groups` attends to."""
    if B % cfg_groups != 0:
        raise ValueError("a batch of %d cannot be split over %d groups" % (B, cfg_groups))
    per = B // cfg_groups
    return slice(group_index * per, (group_index + 1) * per)
