"""The key-set forward (dit_attn_forward_kv) and the context-parallel ring
built on it, on one GPU.  Needs a B200.

* With all keys it is the plain forward, bit for bit; a query subset gives
  the plain forward's rows, bit for bit (every row's arithmetic is its own).
* Key shards: the forward on P key slices (ragged, not tile-aligned), merged
  with dit_attn_merge, meets the BF16 bars against the full-sequence oracle
  (operand-rounded oracle for the bf16 operands; the exact oracle for the
  split form, also on the 2048x2048 outlier workload).
* The ring of context_parallel.ring_attention, each rank emulated in turn on
  the one GPU (the exchange itself runs on gloo ranks in
  tests/test_context_parallel.py).
"""
import numpy as np
import pytest
import torch

import diffusion_transformer_joint_attn_b200 as dit
import workloads as W
from diffusion_transformer_joint_attn_b200 import build, context_parallel as cp

from gpu_cases import (BF16_MAX_ABS, BF16_MEAN_ABS, device_inputs, errors, gather_rows, lse_bound, oracle_rows,
                       rope_tables)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    dit.load_library()


def check(got, lse, rows, O_ref, L_ref, label):
    mx, mean = errors(got, O_ref)
    ratio = float((np.abs(lse - L_ref) / lse_bound(L_ref)).max())
    print("%s: max-abs %.3e mean-abs %.3e max|dLSE|/bound %.3f (%d rows)" % (label, mx, mean, ratio, len(rows)))
    assert mx <= BF16_MAX_ABS and mean <= BF16_MEAN_ABS and ratio <= 1.0, label


@pytest.mark.parametrize("name", ["tiny_256", "t2i_512px"])
def test_all_keys_and_query_subsets_equal_the_plain_forward(name):
    w = W.WORKLOADS[name]
    _, _, _, qd, kd, vd = device_inputs(w)
    c, s = rope_tables(w)
    kr, v16 = torch.empty_like(kd), torch.empty(vd.shape, dtype=torch.float16, device=vd.device)
    dit.dit_attn_prepare_kv(kd, vd, c, s, kr, v16)
    ref, lref = dit.forward(qd, kr, v16, c, s, n_txt=w.n_txt, k_rotated=True, v_f16=True)
    a, la = dit.forward_kv(qd, kr, v16, c, s, k_rotated=True, v_f16=True)
    torch.cuda.synchronize()
    assert torch.equal(a, ref) and torch.equal(la, lref)
    for lo, hi in ((0, 1), (5, 133), (w.N - 77, w.N)):
        qs = qd[:, :, lo:hi].contiguous()
        b, lb = dit.forward_kv(qs, kr, v16, c[lo:hi], s[lo:hi], k_rotated=True, v_f16=True)
        torch.cuda.synchronize()
        assert torch.equal(b, ref[:, :, lo:hi]) and torch.equal(lb, lref[:, :, lo:hi]), (lo, hi)
    assert dit.dit_attn_get_status() == dit.DIT_OK


def _sharded(w, inputs, cuts, split):
    """Merged result of the forward on the key slices [cuts[i], cuts[i+1])."""
    _, _, _, qd, kd, vd = inputs
    c, s = rope_tables(w)
    outs, lses = [], []
    for a, b in zip(cuts[:-1], cuts[1:]):
        block = cp.library_prepare(kd[:, :, a:b].contiguous(), vd[:, :, a:b].contiguous(), c[a:b], s[a:b], split)
        o, l = cp.library_attend(qd, block, c, s, split)
        outs.append(o)
        lses.append(l)
    out, lse = dit.merge(outs, lses, out_f32=True)
    torch.cuda.synchronize()
    assert dit.dit_attn_get_status() == dit.DIT_OK
    return out, lse


@pytest.mark.parametrize("name,cuts", [
    ("t2i_512px", (0, 500, 1100, 1536)),
    ("t2i_1024px_cfg", (0, 1, 129, 2304, 4608)),
])
def test_key_shards_merged_match_the_operand_oracle(name, cuts):
    w = W.WORKLOADS[name]
    inputs = device_inputs(w)
    q, k, v = inputs[:3]
    rows = W.sample_rows(w)
    out, lse = _sharded(w, inputs, cuts, split=False)
    O_op, L_op = oracle_rows(w, q, k, v, rows, operands="bf16")
    check(gather_rows(out, rows), gather_rows(lse, rows), rows, O_op, L_op, name + " %d key shards" % (len(cuts) - 1))


@pytest.mark.parametrize("name,cuts", [
    ("t2i_512px", (0, 700, 1536)),
    ("t2i_2048px", (0, 4224, 8448, 12672, 16896)),
])
def test_split_key_shards_merged_match_the_exact_oracle(name, cuts):
    w = W.WORKLOADS[name]
    inputs = device_inputs(w)
    q, k, v = inputs[:3]
    rows = W.sample_rows(w)
    out, lse = _sharded(w, inputs, cuts, split=True)
    O_ex, L_ex = oracle_rows(w, q, k, v, rows)
    check(gather_rows(out, rows), gather_rows(lse, rows), rows, O_ex, L_ex,
          name + " split, %d key shards" % (len(cuts) - 1))


@pytest.mark.parametrize("P,split", [(2, False), (4, True)])
def test_ring_emulated_rank_by_rank(P, split, monkeypatch):
    """ring_attention's per-rank steps with the library kernels: rank r's
    queries attend to every shard in ring order and merge; the ring's
    exchange is replaced by handing each rank the shard it would receive."""
    w = W.WORKLOADS["t2i_512px"]
    inputs = device_inputs(w)
    q, k, v, qd, kd, vd = inputs
    c, s = rope_tables(w)
    rows = W.sample_rows(w)
    O_ref, L_ref = oracle_rows(w, q, k, v, rows) if split else oracle_rows(w, q, k, v, rows, operands="bf16")
    full = torch.empty(qd.shape, dtype=torch.float32, device=qd.device)
    full_lse = torch.empty(qd.shape[:3], dtype=torch.float32, device=qd.device)
    Ns = w.N // P
    blocks = [cp.library_prepare(kd[:, :, j * Ns:(j + 1) * Ns].contiguous(), vd[:, :, j * Ns:(j + 1) * Ns].contiguous(),
                                 c[j * Ns:(j + 1) * Ns], s[j * Ns:(j + 1) * Ns], split) for j in range(P)]
    for r in range(P):
        mine = cp.token_slice(w.N, r, P)
        step = {"s": 0}

        def exchange(block, rank, size, group):
            step["s"] += 1
            return blocks[(r - step["s"]) % P], []

        monkeypatch.setattr(cp, "_rank_size", lambda group, r=r: (r, P))
        monkeypatch.setattr(cp, "_exchange", exchange)
        monkeypatch.setattr(cp, "library_prepare", lambda *a, r=r: blocks[r])
        o, l = cp.ring_attention(qd[:, :, mine].contiguous(), kd[:, :, mine].contiguous(),
                                 vd[:, :, mine].contiguous(), c, s, split=split, out_f32=True)
        full[:, :, mine] = o
        full_lse[:, :, mine] = l
    torch.cuda.synchronize()
    check(gather_rows(full, rows), gather_rows(full_lse, rows), rows, O_ref, L_ref,
          "ring P=%d%s" % (P, " split" if split else ""))
