"""Context-parallel joint attention: the key/value sequence is sharded over
the ranks of a group, every rank attends its own queries to one key shard
at a time while the shards travel round a ring, and the partial results are
merged through their log-sum-exps.

The pages split the FLUX.1-dev attention over 2 and 4 GPUs this way (context
parallelism, wavespeed.ai "Beschleunigung der FLUX.1-dev Bildgenerierung",
section on context parallelism and First Block Cache).  With P ranks, rank r
holds tokens r N/P .. (r+1) N/P - 1 of q, k and v ([B, H, N/P, D]):

    prepare:  K_r rotated with its own tokens' table rows and V_r in fp16
              (dit_attn_prepare_kv; the split operands of
              dit_attn_prepare_kv_split with split=True), once per call
    step s = 0 .. P-1, block j = (r - s) mod P:
              part_s = dit_attn_forward_kv(q_r, K_j, V_j)   (O_s, LSE_s)
              meanwhile K_j, V_j go to rank r+1 and K_{j-1}, V_{j-1} arrive
              from rank r-1 (NCCL point-to-point send / receive)
    merge:    O_r = sum_s exp(LSE_s - LSE) O_s,  LSE = ln sum_s exp(LSE_s)
              (dit_attn_merge, one launch over the P parts)

Every key is seen exactly once by every query, so the merge is exact
attention over all N keys.  The ring carries each shard P-1 times; the
exchange of step s overlaps the attention of step s.  `prepare`, `attend`
and `merge` may be replaced (the CPU tests run the ring on gloo ranks with
the fp64 oracle in their place).
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist


def _rank_size(group) -> Tuple[int, int]:
    if group is None and not (dist.is_available() and dist.is_initialized()):
        return 0, 1
    return dist.get_rank(group), dist.get_world_size(group)


def token_slice(N: int, rank: int, P: int) -> slice:
    """The tokens rank `rank` of P holds: a contiguous 1/P of the sequence."""
    if N % P != 0:
        raise ValueError("the token count %d is not divisible by the group size %d" % (N, P))
    n = N // P
    return slice(rank * n, (rank + 1) * n)


def library_prepare(k: torch.Tensor, v: torch.Tensor, k_cos, k_sin, split: bool = False) -> List[torch.Tensor]:
    """The key shard's operands for dit_attn_forward_kv: [k_op, v_f16]."""
    from . import dit_attn_prepare_kv, prepare_kv_split
    if split:
        return list(prepare_kv_split(k, v, k_cos, k_sin))
    if k_cos is None:
        return [k.contiguous(), v.to(torch.float16)]
    k_rot = torch.empty_like(k)
    v_f16 = torch.empty(v.shape, dtype=torch.float16, device=v.device)
    dit_attn_prepare_kv(k, v, k_cos, k_sin, k_rot, v_f16)
    return [k_rot, v_f16]


def library_attend(q: torch.Tensor, block: Sequence[torch.Tensor], q_cos, q_sin, split: bool = False):
    """One part: this rank's queries against one prepared key shard, fp32
    output for the merge."""
    from . import forward_kv
    k_op, v_op = block
    return forward_kv(q, k_op, v_op, q_cos, q_sin, out_f32=True, k_rotated=(q_cos is not None and not split),
                      v_f16=True, qk_split=split)


def library_merge(outs: Sequence[torch.Tensor], lses: Sequence[torch.Tensor], out_f32: bool):
    from . import merge
    return merge(list(outs), list(lses), out_f32=out_f32)


def _exchange(block: Sequence[torch.Tensor], rank: int, P: int, group):
    """Start sending `block` to rank+1 and receiving the block of rank-1;
    returns (received tensors, requests)."""
    recv = [torch.empty_like(t) for t in block]
    to, frm = (rank + 1) % P, (rank - 1) % P
    if group is not None:
        to, frm = dist.get_global_rank(group, to), dist.get_global_rank(group, frm)
    ops = []
    for t, r in zip(block, recv):
        ops.append(dist.P2POp(dist.isend, t, to, group))
        ops.append(dist.P2POp(dist.irecv, r, frm, group))
    return recv, dist.batch_isend_irecv(ops)


def ring_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, rope_cos=None, rope_sin=None,
                   group=None, split: bool = False, out_f32: bool = False,
                   prepare: Optional[Callable] = None, attend: Optional[Callable] = None,
                   merge: Optional[Callable] = None):
    """Attention of this rank's token shard of q over all N keys, with the
    key / value shards passed round the ring of `group`.

    q, k, v: this rank's shards [B, H, N/P, D] (bf16 on the GPU path).
    rope_cos / rope_sin: the [N, D/2] tables of the whole sequence, or None.
    split: use the compensated q k^T (DIT_QK_SPLIT).
    Returns (out [B, H, N/P, D], lse [B, H, N/P]) of this rank's queries.
    """
    if q.dim() != 4 or q.shape != k.shape or k.shape != v.shape:
        raise ValueError("q, k, v must be [B, H, N/P, D] shards of one shape")
    rank, P = _rank_size(group)
    if merge is None and P > 16:
        raise ValueError("dit_attn_merge combines at most 16 parts; %d ranks need another merge" % P)
    Ns = k.shape[2]
    N = Ns * P
    if rope_cos is not None and rope_cos.shape[0] != N:
        raise ValueError("the rotary tables must cover all %d tokens" % N)
    mine = token_slice(N, rank, P)
    cos_r = rope_cos[mine] if rope_cos is not None else None
    sin_r = rope_sin[mine] if rope_sin is not None else None
    prepare = prepare or library_prepare
    attend = attend or library_attend
    merge = merge or library_merge
    block = prepare(k, v, cos_r, sin_r, split)
    outs, lses = [], []
    for s in range(P):
        pending = _exchange(block, rank, P, group) if s < P - 1 else None
        o, l = attend(q, block, cos_r, sin_r, split)
        outs.append(o)
        lses.append(l)
        if pending is not None:
            recv, reqs = pending
            for req in reqs:
                req.wait()
            block = recv
    return merge(outs, lses, out_f32)
