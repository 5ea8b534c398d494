"""A layer split by kv head reproduces the whole layer, bit for bit.

The multi-GPU split gives each rank a contiguous range of kv heads (with
their q heads) of a B = 1 layer.  Units share nothing, so the sub-layers,
run through the same C ABI calls on slices of the layer's tensors, must give
exactly the whole layer's selection (counts and index lists) and outputs (O
and LSE).  Here the ranks' sub-layers run one after the other on one GPU.
"""

import numpy as np
import pytest
import torch

import block_sparse_long_sm_b200 as spa
from block_sparse_long_sm_b200.binding import WorkspaceView
from block_sparse_long_sm_b200.shard import rank_sub_layer
from workloads import C1_LLAMA_32K, C3_QWEN_64K, generate

from gpu_common import Run

pytestmark = pytest.mark.gpu


def _filled_lists(p, counts, lists):
    view = WorkspaceView(p, torch.empty(16, dtype=torch.uint8))
    nqb = (p.seq_len + 127) // 128
    out = []
    for h in range(p.heads_q):
        for qb in range(nqb):
            n = int(counts[h * nqb + qb])
            off = view.list_offset(0, h, qb)
            out.append(lists[off:off + n].copy())
    return out


@pytest.mark.parametrize("w,mode,world", [(C1_LLAMA_32K, "anchor", 2), (C1_LLAMA_32K, "sale", 4),
                                          (C3_QWEN_64K.with_(seq_len=16384), "anchor", 2)])
def test_kv_head_split_reproduces_the_layer(w, mode, world):
    inp = generate(w)
    full = Run(inp, mode=mode, sink=w.sink, local=w.local, theta=3.0, tau=0.1,
               block_k=w.block_k if mode == "sale" else None)
    o_full = full.o.clone()
    lse_full = full.lse.clone()
    counts_full = full.counts
    lists_full = _filled_lists(full.params, counts_full, full.lists_host())
    o = torch.full_like(full.o, float("nan"))
    lse = torch.full_like(full.lse, float("nan"))
    nqb = (w.seq_len + 127) // 128
    for rank in range(world):
        sub = rank_sub_layer(full.params, world, rank)
        p = sub.params
        ws = torch.empty(spa.sparse_prefill_workspace_bytes(p), dtype=torch.uint8, device="cuda")
        qp, kp, vp, op, lp = sub.pointers(full.q, full.k, full.v, o, lse)
        spa.check(spa.sparse_prefill_plan(p, qp, kp, ws), "plan")
        spa.check(spa.sparse_prefill_attn(p, qp, kp, vp, ws, op, lp), "attn")
        st, _ = spa.sparse_prefill_stats(p, ws)
        spa.check(st, "stats")
        view = WorkspaceView(p, ws)
        counts = view.counts.cpu().numpy()
        assert np.array_equal(counts, counts_full[sub.h0 * nqb:sub.h1 * nqb]), rank
        lists = _filled_lists(p, counts, view.lists.cpu().numpy())
        for a, b in zip(lists, lists_full[sub.h0 * nqb:sub.h1 * nqb]):
            assert np.array_equal(a, b), rank
    torch.cuda.synchronize()
    assert torch.equal(o.view(torch.int16), o_full.view(torch.int16))
    assert torch.equal(lse.view(torch.int32), lse_full.view(torch.int32))
