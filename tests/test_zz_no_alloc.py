"""The allocation-free selection entry point, sparse_prefill_plan_static.

It serves callers that cannot hand the library a workspace (plugin hosts whose
enqueue step may not allocate, serving stacks that reserve all device memory
at start-up, hot paths where cudaMalloc's possible device synchronisation is
not allowed): its scratch is a fixed device array inside the library.  Here it
is called through the C ABI and its counts and index lists are compared, bit
for bit (integer output), with those of sparse_prefill_plan on the same
inputs, on calls made back to back so that the second call starts from the
first call's leftover scratch.  This file is collected last so that a run that
stops at the first failure has run every other test before it.
"""

import numpy as np
import pytest
import torch

import block_sparse_long_sm_b200 as spa
from block_sparse_long_sm_b200.binding import WorkspaceView, sparse_prefill_plan_static
from workloads import C0_TINY, C1_LLAMA_32K, generate

from gpu_common import to_dev

pytestmark = pytest.mark.gpu


def _reference_plan(p, q, k):
    ws = torch.empty(spa.sparse_prefill_workspace_bytes(p), dtype=torch.uint8, device="cuda")
    spa.check(spa.sparse_prefill_plan(p, q, k, ws), "plan")
    torch.cuda.synchronize()
    view = WorkspaceView(p, ws)
    return view.counts.clone(), view.lists.clone()


def _static_plan(p, q, k, n_lists):
    nqb = (p.seq_len + 127) // 128
    counts = torch.full((p.batch * p.heads_q * nqb,), -1, dtype=torch.int32, device="cuda")
    lists = torch.full((max(n_lists, 1),), -1, dtype=torch.int32, device="cuda")
    err = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    st = sparse_prefill_plan_static(p, q, k, counts, lists, n_lists, err)
    spa.check(st, "plan_static")
    torch.cuda.synchronize()
    return counts, lists[:n_lists], int(err.item())


def _case(w, L, theta, sink, local, step=1):
    inp = generate(w.with_(sink=sink, local=local), seq_len=L)
    q, k = to_dev(inp.q), to_dev(inp.k)
    B, Hq, Hkv = w.batch, w.heads_q, w.heads_kv
    p = spa.make_params(B, Hq, Hkv, L, mode="anchor", sink=sink, local=local, theta=theta,
                        step=step)
    return p, q, k


def _check_same(p, q, k):
    ref_counts, ref_lists = _reference_plan(p, q, k)
    counts, lists, err = _static_plan(p, q, k, ref_lists.numel())
    assert err == 0
    assert torch.equal(counts, ref_counts)
    # compare only the filled prefix of every block's list (the rest is unused capacity)
    view = WorkspaceView(p, torch.empty(spa.sparse_prefill_workspace_bytes(p), dtype=torch.uint8,
                                        device="cuda"))
    c = ref_counts.cpu().numpy()
    a = lists.cpu().numpy()
    b = ref_lists.cpu().numpy()
    nqb = (p.seq_len + 127) // 128
    for bh in range(p.batch * p.heads_q):
        for qb in range(nqb):
            n = int(c[bh * nqb + qb])
            off = view.list_offset(bh // p.heads_q, bh % p.heads_q, qb)
            assert np.array_equal(a[off:off + n], b[off:off + n]), (bh, qb)
    return int(c.sum())


def test_static_plan_matches_workspace_plan_on_back_to_back_calls():
    # call 1: one head, 4K, sparse theta; call 2: GQA 32/8 heads, ragged 3000 rows;
    # call 3: the first problem again, after the second left its scratch behind.
    p1, q1, k1 = _case(C0_TINY, 4096, 2.5, 64, 128)
    kept1 = _check_same(p1, q1, k1)
    p2, q2, k2 = _case(C1_LLAMA_32K, 3000, 3.0, 128, 256)
    kept2 = _check_same(p2, q2, k2)
    assert _check_same(p1, q1, k1) == kept1
    assert kept1 > 0 and kept2 > 0


@pytest.mark.parametrize("step", [2, 3])
def test_static_plan_matches_workspace_plan_with_grouped_query_blocks(step):
    # the workspace plan unions a group of query blocks inside its fused
    # selection kernel when step is a power of two (step 2) and through the
    # separate compaction otherwise (step 3); the static plan always takes
    # the compaction path, over scratch the previous call left behind
    p, q, k = _case(C1_LLAMA_32K, 2500, 3.0, 128, 256, step=step)
    kept = _check_same(p, q, k)
    p1, q1, k1 = _case(C0_TINY, 4096, 2.5, 64, 128, step=step)
    assert _check_same(p1, q1, k1) > 0
    assert _check_same(p, q, k) == kept > 0


def test_static_plan_empty_problem_clears_the_error_word():
    p = spa.make_params(0, 4, 2, 1024, mode="anchor", sink=64, local=128, theta=3.0)
    dummy = torch.empty(16, dtype=torch.int32, device="cuda")
    err = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    assert sparse_prefill_plan_static(p, dummy, dummy, dummy, dummy, 0, err) == spa.SPA_OK
    torch.cuda.synchronize()
    assert int(err.item()) == 0


def test_static_plan_rejects_problems_beyond_its_scratch():
    p = spa.make_params(1, 32, 8, 65536, mode="anchor", sink=128, local=256, theta=5.0)
    dummy = torch.empty(16, dtype=torch.int32, device="cuda")
    st = sparse_prefill_plan_static(p, dummy, dummy, dummy, dummy, 16, None)
    assert st == spa.SPA_ERR_UNSUPPORTED
    p = spa.make_params(1, 1, 1, 4096, mode="sale", sink=64, local=128)
    assert sparse_prefill_plan_static(p, dummy, dummy, dummy, dummy, 16, None) == spa.SPA_ERR_UNSUPPORTED
