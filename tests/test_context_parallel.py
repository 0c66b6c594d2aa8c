"""Context-parallel (ring) attention host logic on gloo ranks on the CPU:
the key / value shards travel round the ring, each rank attends its own
queries to every shard once and merges the parts.  The fp64 oracle stands
in for the three library steps (operand preparation, the per-shard forward
and the merge), so the result must equal the oracle on the full sequence to
rounding; the same ring on the GPU runs the library's kernels
(tests/test_gpu_context_parallel.py)."""
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


def _oracle_steps(scale):
    """prepare / attend / merge of the ring in fp64 with the oracle."""
    import torch
    from oracle import attention as A, merge as M, rope

    def prepare(k, v, cos, sin, split):
        kk = k.double().numpy()
        if cos is not None:
            kk = rope.rotate_with_table(kk, cos.numpy(), sin.numpy())
        return [torch.from_numpy(np.ascontiguousarray(kk)), v.double().contiguous()]

    def attend(q, block, cos, sin, split):
        qq = q.double().numpy()
        if cos is not None:
            qq = rope.rotate_with_table(qq, cos.numpy(), sin.numpy())
        kk, vv = block[0].numpy(), block[1].numpy()
        B, H, Nq, D = qq.shape
        O = np.empty((B, H, Nq, D))
        L = np.empty((B, H, Nq))
        for b in range(B):
            for h in range(H):
                O[b, h], L[b, h] = A.attention_rows(qq[b, h], kk[b, h], vv[b, h], scale)
        return torch.from_numpy(O), torch.from_numpy(L)

    def merge(outs, lses, out_f32):
        B, H, Nq, D = outs[0].shape
        o, l = M.merge([x.reshape(-1, D).numpy() for x in outs], [x.reshape(-1).numpy() for x in lses])
        return torch.from_numpy(o.reshape(B, H, Nq, D)), torch.from_numpy(l.reshape(B, H, Nq))

    return prepare, attend, merge


def _worker(rank, world, port, case, rq):
    import datetime
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import workloads as W
        from diffusion_transformer_joint_attn_b200 import context_parallel as cp
        from oracle import attention as oracle_attention, rope
        result = {}
        if case == "errors":
            def refused(fn):
                try:
                    fn()
                except ValueError:
                    return True
                return False
            x = torch.zeros(1, 2, 4, 8)
            result["shapes"] = refused(lambda: cp.ring_attention(x, x[:, :, :3], x))
            result["tables"] = refused(lambda: cp.ring_attention(x, x, x, torch.zeros(5, 4), torch.zeros(5, 4)))
            result["slice"] = refused(lambda: cp.token_slice(10, 0, 3))
            dist.barrier()
        else:
            rope_on = case == "rope"
            w = W.custom(2, 3, 8 * world, ((4 * world, 6),), outliers=True)
            q, k, v = W.make_qkv(w, seed=7)
            pos = W.positions(w)
            Ns = w.N // world
            mine = cp.token_slice(w.N, rank, world)
            cos = sin = None
            if rope_on:
                c, s = rope.table(pos)
                cos, sin = torch.from_numpy(c), torch.from_numpy(s)
            prepare, attend, merge = _oracle_steps(1.0 / np.sqrt(w.D))
            out, lse = cp.ring_attention(q[:, :, mine], k[:, :, mine], v[:, :, mine], cos, sin, prepare=prepare,
                                         attend=attend, merge=merge)
            O, L = oracle_attention.joint_attention(q, k, v, pos=pos if rope_on else None)
            O = O.reshape(w.B, w.H, w.N, -1)[:, :, mine]
            L = L.reshape(w.B, w.H, w.N)[:, :, mine]
            result["max_err"] = float(np.abs(out.numpy() - O).max() / np.abs(O).max())
            result["lse_err"] = float(np.abs(lse.numpy() - L).max())
            assert out.shape == (w.B, w.H, Ns, w.D)
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


@pytest.mark.parametrize("world,case", [(2, "rope"), (3, "rope"), (4, "plain")])
def test_ring_attention_matches_full_sequence_oracle(world, case):
    res = _run(world, case)
    for rank, r in res.items():
        assert r["max_err"] < 1e-12 and r["lse_err"] < 1e-10, (rank, r)


def test_ring_argument_errors_on_every_rank():
    res = _run(2, "errors")
    for rank, r in res.items():
        assert all(r.values()), (rank, r)


def test_single_process_ring_is_one_part():
    """Without a process group the ring has one rank: one part, merged alone."""
    import torch
    import workloads as W
    from diffusion_transformer_joint_attn_b200 import context_parallel as cp
    from oracle import attention as oracle_attention
    w = W.custom(1, 2, 16, ((4, 4),))
    q, k, v = W.make_qkv(w, seed=2)
    prepare, attend, merge = _oracle_steps(1.0 / np.sqrt(w.D))
    out, lse = cp.ring_attention(q, k, v, prepare=prepare, attend=attend, merge=merge)
    O, L = oracle_attention.joint_attention(q, k, v)
    assert np.abs(out.numpy().reshape(-1, w.D) - O).max() < 1e-12
    assert np.abs(lse.numpy().reshape(-1) - L).max() < 1e-12
    assert cp.token_slice(12, 2, 3) == slice(8, 12)
