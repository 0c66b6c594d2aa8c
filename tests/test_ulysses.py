"""Ulysses sequence parallelism and the CFG batch split (multi-GPU host
logic) on gloo ranks on the CPU.

The exchanges are checked against the full tensors they come from, and the
whole Ulysses attention against the fp64 oracle on the full sequence, with
the oracle standing in for the attention of the local heads (the exchange
logic does not depend on where that attention runs).
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _full(B, H, N, D, seed):
    import torch
    g = torch.Generator().manual_seed(seed)
    return torch.randn(B, H, N, D, generator=g, dtype=torch.float64)


def _worker(rank, world, port, case, rq):
    import datetime
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from diffusion_transformer_joint_attn_b200 import ulysses
        result = {}
        if case == "exchange":
            B, H, N, D = 2, 4 * world, 6 * world, 3
            x = _full(B, H, N, D, 0)
            Ns, Hl = N // world, H // world
            shard = x[:, :, rank * Ns:(rank + 1) * Ns].contiguous()
            heads = ulysses.seq_to_head(shard)
            result["heads_ok"] = bool(torch.equal(heads, x[:, rank * Hl:(rank + 1) * Hl]))
            back = ulysses.head_to_seq(heads)
            result["round_trip_ok"] = bool(torch.equal(back, shard))
            lse = x[..., 0]
            lh = ulysses.head_to_seq(lse[:, rank * Hl:(rank + 1) * Hl].unsqueeze(-1)).squeeze(-1)
            result["lse_ok"] = bool(torch.equal(lh, lse[:, :, rank * Ns:(rank + 1) * Ns]))
        elif case == "errors":
            # every check fails on every rank before a collective is entered
            def refused(fn):
                try:
                    fn()
                except ValueError:
                    return True
                return False
            odd_heads = torch.zeros(1, 2 * world + 1, 4, 3)
            odd_tokens = torch.zeros(1, 1, 2 * world + 1, 3)
            shard = torch.zeros(1, 2 * world, 4, 3)
            result["heads"] = refused(lambda: ulysses.seq_to_head(odd_heads))
            result["tokens"] = refused(lambda: ulysses.head_to_seq(odd_tokens))
            result["tables"] = refused(lambda: ulysses.ulysses_attention(
                shard, shard, shard, torch.zeros(4, 64), torch.zeros(4, 64), attn=lambda *a: None))
            result["shapes"] = refused(lambda: ulysses.ulysses_attention(shard, shard[:, :1], shard))
            result["groups"] = refused(lambda: ulysses.ulysses_attention(shard, shard, shard, head_groups=3,
                                                                         attn=lambda *a: None))
            dist.barrier()                        # the ranks are still in step
        else:
            import workloads as W
            from oracle import attention as oracle_attention
            head_groups = 3 if case == "grouped" else 1
            cfg_groups = 2 if case == "cfg" else 1
            groups = ulysses.cfg_ulysses_groups(world, cfg_groups)
            handles = [dist.new_group(r) for r in groups]          # every rank creates every group, in order
            gi = rank // (world // cfg_groups)
            group = handles[gi]
            P = world // cfg_groups
            r_in = rank % P
            w = W.custom(2 if case == "cfg" else 1, 2 * P * head_groups, 8 * P, ((4 * P, 6),))
            q, k, v = W.make_qkv(w, seed=3)
            pos = W.positions(w)
            share = ulysses.batch_share(w.B, gi, cfg_groups)
            Ns = w.N // P

            def local(t):
                return t[share, :, r_in * Ns:(r_in + 1) * Ns].double().contiguous()

            def oracle_attn(qh, kh, vh, rope_cos, rope_sin, n_txt, out_f32, with_lse):
                O, L = oracle_attention.joint_attention(qh, kh, vh, pos=pos)
                Bl, Hl, N = qh.shape[:3]
                return (torch.from_numpy(O.reshape(Bl, Hl, N, -1)), torch.from_numpy(L.reshape(Bl, Hl, N)))

            cs = torch.zeros(w.N, 64)             # tables of all N tokens (the oracle uses pos)
            calls = []

            def counted(*a):
                calls.append(a[0].shape[1])
                return oracle_attn(*a)
            out, lse = ulysses.ulysses_attention(local(q), local(k), local(v), cs, cs, n_txt=w.n_txt, group=group,
                                                 attn=counted, head_groups=head_groups)
            result["attn_calls"] = calls
            O, L = oracle_attention.joint_attention(q, k, v, pos=pos)
            O = O.reshape(w.B, w.H, w.N, -1)[share, :, r_in * Ns:(r_in + 1) * Ns]
            L = L.reshape(w.B, w.H, w.N)[share, :, r_in * Ns:(r_in + 1) * Ns]
            result["max_err"] = float(np.abs(out.numpy() - O).max())
            result["lse_err"] = float(np.abs(lse.numpy() - L).max())
            for h in handles:
                dist.destroy_process_group(h)
        rq.put((rank, result))
    finally:
        dist.destroy_process_group()


def _run(world, case):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return res


@pytest.mark.parametrize("world", [2, 4])
def test_sequence_head_exchange(world):
    res = _run(world, "exchange")
    for rank, r in res.items():
        assert r["heads_ok"] and r["round_trip_ok"] and r["lse_ok"], (rank, r)


@pytest.mark.parametrize("world", [2, 4])
def test_ulysses_attention_matches_full_sequence_oracle(world):
    res = _run(world, "ulysses")
    for rank, r in res.items():
        assert r["max_err"] < 1e-12 and r["lse_err"] < 1e-12, (rank, r)


@pytest.mark.parametrize("world", [2, 4])
def test_head_group_pipelined_exchanges_match_full_sequence_oracle(world):
    """Three head groups per rank: three attention calls of 2 heads each, and
    the result of the whole-tensor exchange."""
    res = _run(world, "grouped")
    for rank, r in res.items():
        assert r["max_err"] < 1e-12 and r["lse_err"] < 1e-12, (rank, r)
        assert r["attn_calls"] == [2, 2, 2], (rank, r)


def test_exchange_argument_errors_on_every_rank():
    res = _run(2, "errors")
    for rank, r in res.items():
        assert all(r.values()), (rank, r)


def test_cfg_groups_split_the_batch():
    res = _run(4, "cfg")
    for rank, r in res.items():
        assert r["max_err"] < 1e-12 and r["lse_err"] < 1e-12, (rank, r)


def test_group_helpers():
    from diffusion_transformer_joint_attn_b200 import ulysses
    assert ulysses.cfg_ulysses_groups(8, 2) == [[0, 1, 2, 3], [4, 5, 6, 7]]
    assert ulysses.batch_share(2, 1, 2) == slice(1, 2)
    with pytest.raises(ValueError):
        ulysses.cfg_ulysses_groups(6, 4)
