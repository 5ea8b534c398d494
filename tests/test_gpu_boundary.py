"""GPU boundary behaviour: status codes, empty inputs, bounded-wait expiry and
device-side index checks (none of which may fault the GPU)."""

import math

import numpy as np
import pytest
import torch

import block_sparse_long_sm_b200 as spa
from workloads import C0_TINY, generate

from gpu_common import Run, compare_outputs, to_dev

pytestmark = pytest.mark.gpu


def _bufs(L=1024):
    inp = generate(C0_TINY, seq_len=L)
    q, k, v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
    return inp, q, k, v


def test_empty_inputs_are_noops():
    for B, L in ((0, 1024), (1, 0)):
        p = spa.make_params(B, 1, 1, L, sink=64, local=128)
        ws = torch.zeros(spa.sparse_prefill_workspace_bytes(p), dtype=torch.uint8, device="cuda")
        assert spa.sparse_prefill_plan(p, 0, 0, ws) == spa.SPA_OK
        assert spa.sparse_prefill_attn(p, 0, 0, 0, ws, 0) == spa.SPA_OK
        st, s = spa.sparse_prefill_stats(p, ws)
        assert st == spa.SPA_OK and s.kept_pairs == 0


def test_argument_errors_return_before_launch():
    _, q, k, v = _bufs()
    p = spa.make_params(1, 1, 1, 1024, sink=64, local=128)
    n = spa.sparse_prefill_workspace_bytes(p)
    ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    o = torch.empty((1, 1, 1024, 128), dtype=torch.bfloat16, device="cuda")
    assert spa.sparse_prefill_plan(p, q, k, ws, workspace_bytes=n - 1) == spa.SPA_ERR_WORKSPACE
    assert spa.sparse_prefill_plan(p, q, k, 0, workspace_bytes=n) == spa.SPA_ERR_INVALID
    assert spa.sparse_prefill_plan(p, q.data_ptr() + 2, k, ws) == spa.SPA_ERR_INVALID
    assert spa.sparse_prefill_attn(p, q, k, v, ws, 0) == spa.SPA_ERR_INVALID
    bad = [dict(head_dim=64), dict(causal=0), dict(step=0), dict(local=100), dict(local=64),
           dict(theta=math.nan)]
    codes = [spa.SPA_ERR_UNSUPPORTED, spa.SPA_ERR_UNSUPPORTED, spa.SPA_ERR_INVALID,
             spa.SPA_ERR_INVALID, spa.SPA_ERR_INVALID, spa.SPA_ERR_INVALID]
    for kw, code in zip(bad, codes):
        pb = spa.make_params(1, 1, 1, 1024, **{"sink": 64, "local": 128, **kw})
        assert spa.sparse_prefill_plan(pb, q, k, ws) == code, kw
        assert spa.sparse_prefill_workspace_bytes(pb) == 0
    ps = spa.make_params(1, 1, 1, 1024, mode="sale", sink=48, local=128, block_k=32)
    assert spa.sparse_prefill_plan(ps, q, k, ws) == spa.SPA_ERR_UNSUPPORTED
    ps = spa.make_params(1, 1, 1, 1024, mode="sale", sink=64, local=128, tau=0.0)
    assert spa.sparse_prefill_plan(ps, q, k, ws) == spa.SPA_ERR_INVALID


@pytest.mark.parametrize("hq", [1, 2])
def test_bounded_wait_expiry_reports_timeout_and_context_survives(hq):
    """hq = 1 runs the one-head kernel, hq = 2 the paired kernel."""
    from workloads import Workload
    w = Workload(f"stall-{hq}", 11, 1, hq, 1, 1024, sink=64, local=128, needles_per_head=4)
    inp = generate(w)
    q, k, v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
    p = spa.make_params(1, hq, 1, 1024, sink=64, local=128, theta=3.0,
                        wait_limit_us=20000, debug_flags=spa.SPA_DEBUG_STALL_ATTN)
    ws = torch.zeros(spa.sparse_prefill_workspace_bytes(p), dtype=torch.uint8, device="cuda")
    o = torch.zeros((1, hq, 1024, 128), dtype=torch.bfloat16, device="cuda")
    spa.check(spa.sparse_prefill_plan(p, q, k, ws))
    assert spa.sparse_prefill_attn(p, q, k, v, ws, o) == spa.SPA_OK
    st, s = spa.sparse_prefill_stats(p, ws)
    assert st == spa.SPA_ERR_TIMEOUT and (s.error_bits & 1)
    # the context is still usable: a normal call afterwards succeeds and is correct
    run = Run(inp, mode="anchor", sink=64, local=128, theta=3.0, dev=(q, k, v))
    assert run.stats.error_bits == 0
    compare_outputs(run, inp, {(0, h): range(0, 1024, 7) for h in range(hq)})


@pytest.mark.parametrize("hq", [1])
def test_corrupted_list_index_is_caught_in_bounds(hq):
    """A corrupted list entry (out of range) is caught, never followed.  (The
    paired kernel reads the pairs' union lists, an opaque part of the
    workspace; its gather carries the same bounds check.)"""
    from workloads import Workload
    w = Workload(f"corrupt-{hq}", 13, 1, hq, 1, 2048, sink=64, local=128, needles_per_head=8)
    inp = generate(w)
    q, k, v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
    run = Run(inp, mode="anchor", sink=64, local=128, theta=3.2, dev=(q, k, v), do_attn=False)
    kept = [b for b in range(16) if run.counts[run.view.block_index(0, 0, b)] > 0]
    assert kept, "head 0 must keep some candidate"
    qb = kept[-1]
    run.view.lists[run.view.list_offset(0, 0, qb)] = 2048 + 5     # out of range on purpose
    o = torch.zeros((1, hq, 2048, 128), dtype=torch.bfloat16, device="cuda")
    assert spa.sparse_prefill_attn(run.params, q, k, v, run.ws, o) == spa.SPA_OK
    st, s = spa.sparse_prefill_stats(run.params, run.ws)
    assert st == spa.SPA_ERR_INVALID and (s.error_bits & 2)
    torch.cuda.synchronize()
